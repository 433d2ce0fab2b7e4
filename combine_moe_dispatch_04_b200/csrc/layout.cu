// Dispatch layout: per-expert histogram, exclusive prefix sum (ep_send_counts)
// and the two slot maps of assist_info. [combine] Parameters
// (assist_info_for_combine, ep_send_counts, x_active_mask).
//
// The order is a stable counting sort on the key (expert, token, k). Because a
// valid row never repeats an id, a token holds at most one pair per expert,
// and a pair's rank inside its expert's segment is the number of earlier
// tokens routed to that expert. Each warp builds, per expert, a 32-bit mask of
// its lanes (tokens) that route there (shared-memory atomicOr); popcounts of
// those masks give counts and ranks with no ordering race, so the result is
// deterministic.
//
//   BS <= 1024: one CTA of 32 warps does everything (one launch).
//   otherwise : count (one CTA per 256-token tile) -> scatter (same tiles):
//               every scatter CTA sums the per-(tile, expert) counts of the
//               caller's workspace itself (its tile's prefix and the expert
//               totals), scans the totals, and writes its tile's slots; CTA 0
//               also writes the counts and the status word.
#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

// Classifies the K pairs of token t: e[k] = expert id of a routed active
// pair, else -1. Returns the MOE_DEV_* bits of the row.
template <int KM>
__device__ __forceinline__ uint32_t classify_row(const LayoutArgs& a, int t, int (&e)[KM]) {
  const int32_t* row = a.topk_idx + static_cast<size_t>(t) * a.K;
  int ids[KM];
  if ((a.K & 3) == 0 && (reinterpret_cast<uintptr_t>(a.topk_idx) & 15) == 0) {
    // rows of a multiple of 4 ids: 16-byte loads
#pragma unroll
    for (int q = 0; q < KM / 4; ++q) {
      int4 v = make_int4(-1, -1, -1, -1);
      if (4 * q < a.K) v = __ldg(reinterpret_cast<const int4*>(row) + q);
      ids[4 * q] = v.x;
      ids[4 * q + 1] = v.y;
      ids[4 * q + 2] = v.z;
      ids[4 * q + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int k = 0; k < KM; ++k) ids[k] = k < a.K ? __ldg(row + k) : -1;
  }
  uint32_t st = 0;
#pragma unroll
  for (int k = 0; k < KM; ++k) {
    e[k] = -1;
    if (k >= a.K) continue;
    const int id = ids[k];
    if (id < 0 || id >= a.N) {
      st |= MOE_DEV_BAD_ID;
      continue;
    }
    bool dup = false;
#pragma unroll
    for (int j = 0; j < k; ++j) dup |= ids[j] == id;
    if (dup) {
      st |= MOE_DEV_DUP_ID;
      continue;
    }
    if (id < a.E && pair_active(a.mask, a.mask_ndim, t, k, a.K)) e[k] = id;
  }
  return st;
}

// words[warp * E + e] |= bit of this lane, for each routed pair of the lane.
template <int KM>
__device__ __forceinline__ void mark_words(uint32_t* words, int E, const int (&e)[KM], int K) {
  const int warp = threadIdx.x >> 5;
  const uint32_t bit = 1u << (threadIdx.x & 31);
#pragma unroll
  for (int k = 0; k < KM; ++k)
    if (k < K && e[k] >= 0) atomicOr(&words[warp * E + e[k]], bit);
}

// Rank of this lane's token among the tile's tokens routed to expert ex.
__device__ __forceinline__ int tile_rank(const uint32_t* words, int E, int ex) {
  const int warp = threadIdx.x >> 5;
  int r = __popc(words[warp * E + ex] & lanemask_lt());
  for (int w = 0; w < warp; ++w) r += __popc(words[w * E + ex]);
  return r;
}

// Block-wide exclusive scan of one value per thread (blockDim.x <= 1024).
// Returns the exclusive prefix; *total receives the block total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  int inc = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    int n = __shfl_up_sync(0xFFFFFFFFu, inc, d);
    if (lane >= d) inc += n;
  }
  if (lane == 31) warp_sums[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int s = lane < nwarps ? warp_sums[lane] : 0;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      int n = __shfl_up_sync(0xFFFFFFFFu, s, d);
      if (lane >= d) s += n;
    }
    if (lane < nwarps) warp_sums[lane] = s;  // inclusive warp prefix
  }
  __syncthreads();
  const int before = warp == 0 ? 0 : warp_sums[warp - 1];
  *total = warp_sums[nwarps - 1];
  return before + inc - v;
}

// Writes both halves of assist_info for token t's pairs given their slots.
template <int KM>
__device__ __forceinline__ void write_slots(const LayoutArgs& a, int t, const int (&e)[KM],
                                            const int (&slot)[KM]) {
  const size_t A = static_cast<size_t>(a.A);
#pragma unroll
  for (int k = 0; k < KM; ++k) {
    if (k >= a.K) continue;
    const int tk = t * a.K + k;
    if (e[k] >= 0) a.assist[slot[k]] = tk;
    a.assist[A + tk] = e[k] >= 0 ? slot[k] : -1;
  }
}

// ---------------------------------------------------------------------------
// One-CTA layout for BS <= 1024: 32 warps, one token per thread.
// Dynamic shared memory: words[32][E].
template <int KM>
__global__ void __launch_bounds__(1024) layout_small_kernel(LayoutArgs a) {
  extern __shared__ uint32_t words[];
  __shared__ int offs[1024];
  __shared__ int warp_sums[32];
  __shared__ uint32_t status;
  pdl_trigger();
  pdl_wait();
  const int E = a.E;
  for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) words[i] = 0;
  if (threadIdx.x == 0) status = 0;
  __syncthreads();

  const int t = threadIdx.x;
  int e[KM];
  uint32_t st = 0;
  if (t < a.bs) {
    st = classify_row<KM>(a, t, e);
    mark_words<KM>(words, E, e, a.K);
  } else {
#pragma unroll
    for (int k = 0; k < KM; ++k) e[k] = -1;
  }
  if (st) atomicOr(&status, st);
  __syncthreads();

  int cnt = 0;
  if (threadIdx.x < E)
    for (int w = 0; w < 32; ++w) cnt += __popc(words[w * E + threadIdx.x]);
  int total;
  const int excl = block_exclusive_scan(cnt, warp_sums, &total);
  if (threadIdx.x < E) {
    offs[threadIdx.x] = excl;
    a.expert_token_nums[threadIdx.x] = cnt;
    a.ep_send_counts[threadIdx.x] = excl;
  }
  if (threadIdx.x == 0) a.ep_send_counts[E] = total;
  __syncthreads();

  if (t < a.bs) {
    int slot[KM];
#pragma unroll
    for (int k = 0; k < KM; ++k)
      slot[k] = (k < a.K && e[k] >= 0) ? offs[e[k]] + tile_rank(words, E, e[k]) : -1;
    write_slots<KM>(a, t, e, slot);
  }
  for (int s = total + threadIdx.x; s < a.A; s += blockDim.x) a.assist[s] = -1;
  if (threadIdx.x == 0 && a.dev_status) *a.dev_status = status;
}

// ---------------------------------------------------------------------------
// Fused dispatch for BS <= 1024 (layout + permute in one launch). Every CTA
// rebuilds the whole layout in shared memory exactly as layout_small_kernel
// does (the ids are at most 64 KB and sit in L2), CTA 0 alone writes the
// layout's outputs, and CTA c copies the rows of tokens [c * per, (c+1) * per)
// to their slots: one thread per 16-byte vector, read once, stored K times.
// Dynamic shared memory: words[32][E].
template <int KM>
__global__ void __launch_bounds__(1024) dispatch_small_kernel(LayoutArgs a, const uint4* x,
                                                              uint4* expand_x, int V, int per) {
  extern __shared__ uint32_t words[];
  __shared__ int offs[1024];
  __shared__ int warp_sums[32];
  __shared__ uint32_t status;
  __shared__ int slot_sh[kLayoutSmallMaxTokens / 8][KM];  // slots of this CTA's tokens
  pdl_trigger();
  pdl_wait();
  const int E = a.E;
  const bool writer = blockIdx.x == 0;
  for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) words[i] = 0;
  if (threadIdx.x == 0) status = 0;
  __syncthreads();
  const int t = threadIdx.x;
  int e[KM];
  uint32_t st = 0;
  if (t < a.bs) {
    st = classify_row<KM>(a, t, e);
    mark_words<KM>(words, E, e, a.K);
  } else {
#pragma unroll
    for (int k = 0; k < KM; ++k) e[k] = -1;
  }
  if (st) atomicOr(&status, st);
  __syncthreads();
  int cnt = 0;
  if (threadIdx.x < E)
    for (int w = 0; w < 32; ++w) cnt += __popc(words[w * E + threadIdx.x]);
  int total;
  const int excl = block_exclusive_scan(cnt, warp_sums, &total);
  if (threadIdx.x < E) {
    offs[threadIdx.x] = excl;
    if (writer) {
      a.expert_token_nums[threadIdx.x] = cnt;
      a.ep_send_counts[threadIdx.x] = excl;
    }
  }
  if (writer && threadIdx.x == 0) a.ep_send_counts[E] = total;
  __syncthreads();
  const int t0 = blockIdx.x * per;
  if (t < a.bs) {
    int slot[KM];
#pragma unroll
    for (int k = 0; k < KM; ++k)
      slot[k] = (k < a.K && e[k] >= 0) ? offs[e[k]] + tile_rank(words, E, e[k]) : -1;
    if (writer) write_slots<KM>(a, t, e, slot);
    if (t >= t0 && t < t0 + per) {
#pragma unroll
      for (int k = 0; k < KM; ++k)
        if (k < a.K) slot_sh[t - t0][k] = slot[k];
    }
  }
  if (writer) {
    for (int s = total + threadIdx.x; s < a.A; s += blockDim.x) a.assist[s] = -1;
    if (threadIdx.x == 0 && a.dev_status) *a.dev_status = status;
  }
  __syncthreads();
  const int t1 = min(a.bs, t0 + per);
  for (int i = threadIdx.x; i < (t1 - t0) * V; i += blockDim.x) {
    const int tl = i / V;
    const int v = i - tl * V;
    const uint4 val = ld_nc_v4(x + static_cast<size_t>(t0 + tl) * V + v);
    for (int k = 0; k < a.K; ++k) {
      const int s = slot_sh[tl][k];
      if (s >= 0) st_v4(expand_x + static_cast<size_t>(s) * V + v, val);
    }
  }
}

// ---------------------------------------------------------------------------
// Multi-CTA layout. Workspace: tile_counts[T][E] int32, then tile_status[T].

struct TileWs {
  int32_t* counts;
  uint32_t* status;
};

__device__ __forceinline__ TileWs tile_ws(const LayoutArgs& a, int T) {
  TileWs w;
  w.counts = static_cast<int32_t*>(a.workspace);
  w.status = reinterpret_cast<uint32_t*>(w.counts + static_cast<size_t>(T) * a.E);
  return w;
}

constexpr int kTileWarps = kLayoutTileTokens / 32;

// Phase 1: per-tile expert counts and status bits.
template <int KM>
__global__ void __launch_bounds__(kLayoutTileTokens) layout_count_kernel(LayoutArgs a, int T) {
  extern __shared__ uint32_t words[];  // [kTileWarps][E]
  __shared__ uint32_t status;
  pdl_trigger();
  pdl_wait();
  const int E = a.E;
  for (int i = threadIdx.x; i < kTileWarps * E; i += blockDim.x) words[i] = 0;
  if (threadIdx.x == 0) status = 0;
  __syncthreads();
  const int t = blockIdx.x * kLayoutTileTokens + threadIdx.x;
  if (t < a.bs) {
    int e[KM];
    const uint32_t st = classify_row<KM>(a, t, e);
    mark_words<KM>(words, E, e, a.K);
    if (st) atomicOr(&status, st);
  }
  __syncthreads();
  TileWs ws = tile_ws(a, T);
  for (int ex = threadIdx.x; ex < E; ex += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kTileWarps; ++w) c += __popc(words[w * E + ex]);
    ws.counts[static_cast<size_t>(blockIdx.x) * E + ex] = c;
  }
  if (threadIdx.x == 0) ws.status[blockIdx.x] = status;
}

// Phase 2 for one 256-token tile, run by a whole CTA: the tile's first slot
// per expert from the count matrix (prefix over earlier tiles + exclusive
// scan of the expert totals), then slot[] of this thread's token (t < BS).
// The CTA with first_cta writes the counts, prefix sums and status word.
// Shared memory (dynamic): words[kTileWarps][E], base[E], total[E], and two
// [G][E] partial-sum arrays (G * E <= blockDim).
template <int KM>
__device__ __forceinline__ void tile_slots(const LayoutArgs& a, int T, int tile, bool first_cta,
                                           uint32_t* smem, int* warp_sums, uint32_t* status,
                                           int (&e)[KM], int (&slot)[KM], int* grand_out) {
  const int E = a.E;
  uint32_t* words = smem;
  int* base = reinterpret_cast<int*>(smem + kTileWarps * E);
  int* total = base + E;
  for (int i = threadIdx.x; i < kTileWarps * E; i += blockDim.x) words[i] = 0;
  if (threadIdx.x == 0) *status = 0;
  // this thread's token: its ids are loaded now, so their latency overlaps
  // the count-matrix loads below
  const int t = tile * kLayoutTileTokens + threadIdx.x;
#pragma unroll
  for (int k = 0; k < KM; ++k) e[k] = -1;
  if (t < a.bs) classify_row<KM>(a, t, e);
  const TileWs ws = tile_ws(a, T);
  // Sum the count matrix over tiles: G groups of E threads split the tiles
  // (G = 1 when E >= blockDim), then one thread per expert adds the groups.
  const int G = E < static_cast<int>(blockDim.x) ? blockDim.x / E : 1;
  int* part_before = total + E;         // [G][E]
  int* part_all = part_before + G * E;  // [G][E]
  if (G > 1) {
    const int g = threadIdx.x / E, ex = threadIdx.x - g * E;
    if (g < G) {
      int before = 0, all = 0;
#pragma unroll 4
      for (int i = g; i < T; i += G) {
        const int c = ws.counts[static_cast<size_t>(i) * E + ex];
        before += i < tile ? c : 0;
        all += c;
      }
      part_before[g * E + ex] = before;
      part_all[g * E + ex] = all;
    }
    __syncthreads();
    for (int ex2 = threadIdx.x; ex2 < E; ex2 += blockDim.x) {
      int before = 0, all = 0;
      for (int gg = 0; gg < G; ++gg) {
        before += part_before[gg * E + ex2];
        all += part_all[gg * E + ex2];
      }
      base[ex2] = before;
      total[ex2] = all;
    }
  } else {
    for (int ex = threadIdx.x; ex < E; ex += blockDim.x) {
      int before = 0, all = 0;
#pragma unroll 8
      for (int i = 0; i < T; ++i) {
        const int c = ws.counts[static_cast<size_t>(i) * E + ex];
        before += i < tile ? c : 0;
        all += c;
      }
      base[ex] = before;
      total[ex] = all;
    }
  }
  if (first_cta) {
    uint32_t st = 0;
    for (int i = threadIdx.x; i < T; i += blockDim.x) st |= ws.status[i];
    if (st) atomicOr(status, st);
  }
  __syncthreads();
  // exclusive scan of total[0, E): each thread owns a contiguous run of experts
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = min(E, static_cast<int>(threadIdx.x) * per), e1 = min(E, e0 + per);
  int run = 0;
  for (int ex = e0; ex < e1; ++ex) run += total[ex];
  int grand;
  int off = block_exclusive_scan(run, warp_sums, &grand);
  for (int ex = e0; ex < e1; ++ex) {
    const int c = total[ex];
    if (first_cta) {
      a.expert_token_nums[ex] = c;
      a.ep_send_counts[ex] = off;
    }
    base[ex] += off;
    off += c;
  }
  if (first_cta && threadIdx.x == 0) {
    a.ep_send_counts[E] = grand;
    if (a.dev_status) *a.dev_status = *status;
  }
  if (t < a.bs) mark_words<KM>(words, E, e, a.K);  // words were zeroed before the syncs above
  __syncthreads();
#pragma unroll
  for (int k = 0; k < KM; ++k)
    slot[k] = (t < a.bs && k < a.K && e[k] >= 0) ? base[e[k]] + tile_rank(words, E, e[k]) : -1;
  *grand_out = grand;
}

// Phase 2 as its own launch: every tile's slots, and -1 for the unused
// slots [R, A).
template <int KM>
__global__ void __launch_bounds__(kLayoutTileTokens) layout_scatter_kernel(LayoutArgs a, int T) {
  extern __shared__ uint32_t smem[];
  __shared__ int warp_sums[32];
  __shared__ uint32_t status;
  pdl_trigger();
  pdl_wait();
  int e[KM], slot[KM], grand;
  tile_slots<KM>(a, T, blockIdx.x, blockIdx.x == 0, smem, warp_sums, &status, e, slot, &grand);
  const int t = blockIdx.x * kLayoutTileTokens + threadIdx.x;
  if (t < a.bs) write_slots<KM>(a, t, e, slot);
  for (int s = grand + blockIdx.x * blockDim.x + threadIdx.x; s < a.A;
       s += gridDim.x * blockDim.x)
    a.assist[s] = -1;
}

template <int KM>
cudaError_t launch_dispatch_small_k(const LayoutArgs& a, const void* x, void* expand_x, int H,
                                    cudaStream_t st) {
  const int V = H / kVecElems;
  // at most kLayoutSmallMaxTokens / 8 tokens per CTA (the slot buffer's size)
  int blocks = sm_count();
  if (blocks > a.bs) blocks = a.bs > 0 ? a.bs : 1;
  int per = (a.bs + blocks - 1) / blocks;
  if (per > kLayoutSmallMaxTokens / 8) per = kLayoutSmallMaxTokens / 8;
  if (per < 1) per = 1;
  blocks = a.bs > 0 ? (a.bs + per - 1) / per : 1;
  const size_t smem = 32u * a.E * sizeof(uint32_t);
  if (smem > 32 * 1024) {  // with the static buffers: opt in before the total passes 48 KB
    cudaError_t err = cudaFuncSetAttribute(dispatch_small_kernel<KM>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
  }
  return launch_pdl(dispatch_small_kernel<KM>, dim3(blocks), dim3(1024), smem, st, a,
                    static_cast<const uint4*>(x), static_cast<uint4*>(expand_x), V, per);
}

template <int KM>
cudaError_t launch_layout_k(const LayoutArgs& a, cudaStream_t st) {
  if (a.bs <= kLayoutSmallMaxTokens) {
    const size_t smem = 32u * a.E * sizeof(uint32_t);
    if (smem > 32 * 1024) {
      cudaError_t err = cudaFuncSetAttribute(layout_small_kernel<KM>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
      if (err != cudaSuccess) return err;
    }
    return launch_pdl(layout_small_kernel<KM>, dim3(1), dim3(1024), smem, st, a);
  }
  const int T = (a.bs + kLayoutTileTokens - 1) / kLayoutTileTokens;
  const size_t smem_count = static_cast<size_t>(kTileWarps) * a.E * sizeof(uint32_t);
  const size_t smem_scatter =
      smem_count + 2u * a.E * sizeof(int) + 2u * kLayoutTileTokens * sizeof(int);
  cudaError_t err = launch_pdl(layout_count_kernel<KM>, dim3(T), dim3(kLayoutTileTokens),
                               smem_count, st, a, T);
  if (err != cudaSuccess) return err;
  return launch_pdl(layout_scatter_kernel<KM>, dim3(T), dim3(kLayoutTileTokens), smem_scatter,
                    st, a, T);
}

}  // namespace

cudaError_t launch_dispatch_small(const LayoutArgs& a, const void* x, void* expand_x, int H,
                                  cudaStream_t st) {
  if (a.K <= 2) return launch_dispatch_small_k<2>(a, x, expand_x, H, st);
  if (a.K <= 4) return launch_dispatch_small_k<4>(a, x, expand_x, H, st);
  if (a.K <= 8) return launch_dispatch_small_k<8>(a, x, expand_x, H, st);
  return launch_dispatch_small_k<16>(a, x, expand_x, H, st);
}

size_t layout_workspace_bytes(int bs, int E) {
  if (bs <= kLayoutSmallMaxTokens) return 0;
  const size_t T = (static_cast<size_t>(bs) + kLayoutTileTokens - 1) / kLayoutTileTokens;
  return T * static_cast<size_t>(E) * 4 + T * 4;
}

cudaError_t launch_layout(const LayoutArgs& a, cudaStream_t st) {
  if (a.K <= 2) return launch_layout_k<2>(a, st);
  if (a.K <= 4) return launch_layout_k<4>(a, st);
  if (a.K <= 8) return launch_layout_k<8>(a, st);
  return launch_layout_k<16>(a, st);
}

}  // namespace moe
