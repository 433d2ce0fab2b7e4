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
//   BS <= 16384 (and the masks fit in shared memory): one launch of a
//               thread-block cluster of up to 8 CTAs of 1024 threads. Each CTA
//               counts its tokens, scans its per-warp counts per expert, and
//               publishes its per-expert totals; after one cluster barrier
//               every CTA reads the others' totals from distributed shared
//               memory, scans the grand totals and writes its tokens' slots.
//               No workspace.
//   otherwise : count (one CTA per 256-token tile) -> column scan (the count
//               matrix's exclusive prefix over tiles, in place, and the expert
//               totals) -> scatter (same tiles): O(tiles * E) work in all.
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
  // the mask is loaded with the ids, not after them (one DRAM round trip)
  bool act[KM];
#pragma unroll
  for (int k = 0; k < KM; ++k) act[k] = k < a.K && pair_active(a.mask, a.mask_ndim, t, k, a.K);
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
    if (id < a.E && act[k]) e[k] = id;
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

// The same for two values per thread at once (one pass of barriers).
__device__ __forceinline__ int2 block_exclusive_scan2(int2 v, int2* warp_sums, int2* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  int2 inc = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int nx = __shfl_up_sync(0xFFFFFFFFu, inc.x, d);
    const int ny = __shfl_up_sync(0xFFFFFFFFu, inc.y, d);
    if (lane >= d) {
      inc.x += nx;
      inc.y += ny;
    }
  }
  if (lane == 31) warp_sums[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int2 s = lane < nwarps ? warp_sums[lane] : make_int2(0, 0);
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int nx = __shfl_up_sync(0xFFFFFFFFu, s.x, d);
      const int ny = __shfl_up_sync(0xFFFFFFFFu, s.y, d);
      if (lane >= d) {
        s.x += nx;
        s.y += ny;
      }
    }
    if (lane < nwarps) warp_sums[lane] = s;  // inclusive warp prefix
  }
  __syncthreads();
  const int2 before = warp == 0 ? make_int2(0, 0) : warp_sums[warp - 1];
  *total = warp_sums[nwarps - 1];
  return make_int2(before.x + inc.x - v.x, before.y + inc.y - v.y);
}


// ---------------------------------------------------------------------------
// Cluster layout. CTA r of the cluster (CS <= 8 CTAs of 1024 threads) takes the
// tokens [r P, (r + 1) P), P = TPT * 1024, as TPT sub-blocks of 32 warps x 32
// lanes. Dynamic shared memory: words[TPT][32][S] (lane masks per warp and
// expert, S = E | 1 so a warp's column reads hit 32 different banks),
// pre[TPT][32][S] uint16 (exclusive prefix of the mask popcounts over the
// CTA's warps, per expert), tot[E] (this CTA's per-expert totals, read by the
// other CTAs of the cluster) and base[E] (first slot of this CTA's pairs per
// expert).

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
// Cluster-wide barrier halves (every thread of every CTA of the cluster).
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// First half of a cluster barrier that orders nothing (this CTA has started),
// and the matching wait.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
// Stores v into the shared memory of CTA `rank` of this cluster, at the
// position of `local` in this CTA's shared memory.
__device__ __forceinline__ void st_dsmem_u32(void* local, uint32_t rank, uint32_t v) {
  const uint32_t addr = static_cast<uint32_t>(__cvta_generic_to_shared(local));
  uint32_t raddr;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(raddr) : "r"(addr), "r"(rank));
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(raddr), "r"(v) : "memory");
}
// A 32-bit word of the shared memory of CTA `rank` of this cluster, at the
// position of `local` in this CTA's shared memory.
__device__ __forceinline__ uint32_t ld_dsmem_u32(const void* local, uint32_t rank) {
  const uint32_t addr = static_cast<uint32_t>(__cvta_generic_to_shared(local));
  uint32_t raddr, v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(raddr) : "r"(addr), "r"(rank));
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(raddr) : "memory");
  return v;
}

__host__ __device__ constexpr int cluster_stride(int E) { return E | 1; }

constexpr int kClusterMaxCtas = 16;  // blocks per cluster, at most

// Per (sub-block, warp, expert): the lane mask of the warp's tokens routed to
// the expert (x) and the number of the CTA's earlier tokens routed there (y).
// One 8-byte entry, so a pair's rank is one shared-memory load.
struct alignas(8) MaskPre {
  uint32_t mask;
  uint32_t pre;
};
// Per expert: the first slot of this CTA's pairs (x) and their start in the
// CTA's expert-ordered pair list (y).
struct alignas(8) BaseOfs {
  int first;
  int lofs;
};

// mp[tpt][nt / 32][S], bo[E], tot[E] (cluster kernel and fused dispatch, nt
// threads); the cluster kernel also keeps its pairs in expert order,
// ltk[tpt * nt * K], and when `flat`, each list entry's expert,
// lex[tpt * nt * K] (16-bit).
__host__ __device__ constexpr size_t cluster_smem_bytes(int E, int tpt, int nt = 1024) {
  return static_cast<size_t>(tpt) * (nt / 32) * cluster_stride(E) * sizeof(MaskPre) +
         static_cast<size_t>(E) * (4 + sizeof(BaseOfs));
}
__host__ __device__ constexpr size_t cluster_kernel_smem_bytes(int E, int tpt, int K, int nt,
                                                               bool flat = false) {
  return cluster_smem_bytes(E, tpt, nt) + static_cast<size_t>(tpt) * nt * K * (flat ? 6 : 4);
}

// The slot -> pair half of assist_info for a block's routed pairs, written run
// by run: the block's pairs of expert e take the consecutive slots
// [first[e], first[e] + count[e]), and ltk[lofs[e] + r] holds t * K + k of the
// one of rank r, so every warp (experts w, w + 32, ...) writes contiguous ints.
__device__ __forceinline__ void write_runs(const LayoutArgs& a, const int* first, const int* count,
                                           const int* lofs, const int* ltk, int stride) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  for (int ex = warp; ex < a.E; ex += nwarps) {
    const int n = count[ex], f = first[ex * stride], l = lofs[ex * stride];
    for (int j = lane; j < n; j += 32) a.assist[f + j] = ltk[l + j];
  }
}

// The same from a list that also records each entry's expert (lex[p]): thread
// i writes list positions i, i + NT, ... (four loads in flight), so
// neighbouring threads write neighbouring slots however short the runs are.
__device__ __forceinline__ void write_flat(const LayoutArgs& a, const BaseOfs* bo,
                                           const uint16_t* lex, const int* ltk, int n) {
  const int nt = static_cast<int>(blockDim.x);
  for (int p0 = threadIdx.x; p0 < n; p0 += 4 * nt) {
    int v[4], s[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int p = p0 + q * nt;
      s[q] = -1;
      if (p < n) {
        const BaseOfs b = bo[lex[p]];
        s[q] = b.first + (p - b.lofs);
        v[q] = ltk[p];
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (s[q] >= 0) a.assist[s[q]] = v[q];
  }
}

// Token t's K pair -> slot entries (assist[A + t K + k]), with 16- or 8-byte
// stores when K and A allow them (K consecutive ints per thread).
template <int KM>
__device__ __forceinline__ void store_pair_slots(const LayoutArgs& a, int t, const int (&slot)[KM]) {
  int* dst = a.assist + static_cast<size_t>(a.A) + static_cast<size_t>(t) * a.K;
  const uintptr_t addr = reinterpret_cast<uintptr_t>(dst);
  if (KM >= 4 && (a.K & 3) == 0 && (addr & 15) == 0) {
#pragma unroll
    for (int q = 0; q < KM / 4; ++q)
      if (4 * q < a.K)
        reinterpret_cast<int4*>(dst)[q] =
            make_int4(slot[4 * q], slot[4 * q + 1], slot[4 * q + 2], slot[4 * q + 3]);
  } else if (KM >= 2 && (a.K & 1) == 0 && (addr & 7) == 0) {
#pragma unroll
    for (int q = 0; q < KM / 2; ++q)
      if (2 * q < a.K) reinterpret_cast<int2*>(dst)[q] = make_int2(slot[2 * q], slot[2 * q + 1]);
  } else {
#pragma unroll
    for (int k = 0; k < KM; ++k)
      if (k < a.K) dst[k] = slot[k];
  }
}

// Writes both halves of assist_info for token t's pairs given their slots (-1
// for a pair that is not routed).
template <int KM>
__device__ __forceinline__ void write_slots(const LayoutArgs& a, int t, const int (&slot)[KM]) {
#pragma unroll
  for (int k = 0; k < KM; ++k)
    if (k < a.K && slot[k] >= 0) a.assist[slot[k]] = t * a.K + k;
  store_pair_slots<KM>(a, t, slot);
}

// Counts this CTA's tokens [t0, t0 + TPT * NT) (one per thread and sub-block)
// into the lane masks, then per expert the exclusive prefix of the popcounts
// over (sub-block, warp) into mp[].pre and the CTA's total into tot (thread e
// takes expert e's column). mp must be zero on entry; e receives each token's
// routed experts (-1 elsewhere) and the status bits are ORed into *status.
template <int KM, int TPT, int NT>
__device__ __forceinline__ void cta_count_scan(const LayoutArgs& a, int t0, int S, MaskPre* mp,
                                               int* tot, uint32_t* status, int (&e)[TPT][KM]) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t st = 0;
#pragma unroll
  for (int i = 0; i < TPT; ++i) {
    const int t = t0 + i * NT + threadIdx.x;
    if (t < a.bs) {
      st |= classify_row<KM>(a, t, e[i]);
      const uint32_t bit = 1u << lane;
#pragma unroll
      for (int k = 0; k < KM; ++k)
        if (k < a.K && e[i][k] >= 0) atomicOr(&mp[(i * NW + warp) * S + e[i][k]].mask, bit);
    } else {
#pragma unroll
      for (int k = 0; k < KM; ++k) e[i][k] = -1;
    }
  }
  if (st) atomicOr(status, st);
  __syncthreads();
  // one thread per expert column (E <= NT): its popcounts over (sub-block,
  // warp), eight entries loaded together at a time, their running sum stored as
  // each entry's prefix, and the CTA's total
  if (static_cast<int>(threadIdx.x) < a.E) {
    const int ex = threadIdx.x;
    constexpr int N = TPT * NW, CH = N < 8 ? N : 8;
    int run = 0;
#pragma unroll
    for (int i0 = 0; i0 < N; i0 += CH) {
      int c[CH];
#pragma unroll
      for (int i = 0; i < CH; ++i) c[i] = __popc(mp[(i0 + i) * S + ex].mask);
#pragma unroll
      for (int i = 0; i < CH; ++i) {
        mp[(i0 + i) * S + ex].pre = static_cast<uint32_t>(run);
        run += c[i];
      }
    }
    tot[ex] = run;
  }
}

// Rank among the CTA's pairs of expert ex of this thread's token (sub-block i).
template <int NT>
__device__ __forceinline__ int cta_rank(const MaskPre* mp, int i, int S, int ex) {
  const MaskPre m = mp[(i * (NT / 32) + (threadIdx.x >> 5)) * S + ex];
  return static_cast<int>(m.pre) + __popc(m.mask & lanemask_lt());
}

// Two ways to exchange the per-expert totals. With `push` (when cs * E + 16
// ints fit in the pair-list area, which is not yet in use), every CTA stores
// its totals (and its status word, for CTA 0) into every CTA's shared memory
// before one cluster barrier, after which all reads are local; a first
// barrier, arrived at on entry, makes sure every CTA has started before any
// store reaches it. Otherwise each CTA loads the others' totals after the
// barrier, and a second barrier keeps every CTA alive until those loads are
// done.
template <int KM, int TPT, int NT>
__global__ void __launch_bounds__(NT, 1) layout_cluster_kernel(LayoutArgs a, int flat, int push) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int2 warp_sums2[32];
  __shared__ uint32_t status, status_all;
  const int E = a.E;
  const int S = cluster_stride(E);
  MaskPre* mp = reinterpret_cast<MaskPre*>(smem);
  BaseOfs* bo = reinterpret_cast<BaseOfs*>(smem + static_cast<size_t>(TPT) * (NT / 32) * S *
                                                      sizeof(MaskPre));
  int* tot = reinterpret_cast<int*>(bo + E);
  int* ltk = tot + E;
  uint16_t* lex = reinterpret_cast<uint16_t*>(ltk + TPT * NT * a.K);  // when flat
  const uint32_t rank = cluster_ctarank(), cs = cluster_nctarank();
  int* xch = ltk;           // push: [cs][E] totals, then [cs] status words
  int* xst = ltk + cs * E;  //   (the pair list is written only after they are read)
  pdl_trigger();
  if (push) cluster_arrive_relaxed();  // this CTA has started
  for (int i = threadIdx.x; i < TPT * (NT / 32) * S; i += NT) mp[i] = MaskPre{0u, 0u};
  if (threadIdx.x == 0) {
    status = 0;
    status_all = 0;
  }
  __syncthreads();
  pdl_wait();

  const int t0 = static_cast<int>(rank) * TPT * NT;
  int e[TPT][KM];
  cta_count_scan<KM, TPT, NT>(a, t0, S, mp, tot, &status, e);
  int grand = 0, before = 0;
  uint32_t cst = 0;
  if (push) {
    __syncwarp();
    cluster_wait_acquire();  // every CTA of the cluster has started
    if (threadIdx.x < E) {
      const uint32_t mine = static_cast<uint32_t>(tot[threadIdx.x]);
      for (uint32_t c = 0; c < cs; ++c) st_dsmem_u32(xch + rank * E + threadIdx.x, c, mine);
    }
    if (threadIdx.x == 0) st_dsmem_u32(xst + rank, 0, status);
    __syncwarp();
    cluster_arrive_release();  // the stores are published to the cluster
    cluster_wait_acquire();
    if (threadIdx.x < E) {
      for (int c = 0; c < static_cast<int>(cs); ++c) {
        const int v = xch[c * E + threadIdx.x];
        grand += v;
        before += c < static_cast<int>(rank) ? v : 0;
      }
    }
    if (rank == 0 && threadIdx.x < cs) cst = static_cast<uint32_t>(xst[threadIdx.x]);
  } else {
    __syncwarp();
    cluster_arrive_release();  // tot and status are published to the cluster
    cluster_wait_acquire();
    // grand totals and the pairs of the CTAs before this one, per expert (all
    // the remote loads are issued before any is used)
    if (threadIdx.x < E) {
      int v[kClusterMaxCtas];
#pragma unroll
      for (int c = 0; c < kClusterMaxCtas; ++c)
        v[c] = c < static_cast<int>(cs) ? static_cast<int>(ld_dsmem_u32(tot + threadIdx.x, c)) : 0;
#pragma unroll
      for (int c = 0; c < kClusterMaxCtas; ++c) {
        grand += v[c];
        before += c < static_cast<int>(rank) ? v[c] : 0;
      }
    }
    if (rank == 0 && threadIdx.x < cs) cst = ld_dsmem_u32(&status, threadIdx.x);
    __syncwarp();
    cluster_arrive_release();  // done reading the other CTAs' shared memory
  }
  if (cst) atomicOr(&status_all, cst);
  // exclusive scans over the experts of the grand totals (global first slots) and
  // of this CTA's totals (positions in its expert-ordered pair list)
  int2 totals;
  const int2 ex2 = block_exclusive_scan2(
      threadIdx.x < E ? make_int2(grand, tot[threadIdx.x]) : make_int2(0, 0), warp_sums2, &totals);
  const int total = totals.x, listed = totals.y;
  const int excl = ex2.x, lexcl = ex2.y;
  if (threadIdx.x < E) {
    bo[threadIdx.x] = BaseOfs{excl + before, lexcl};
    if (rank == 0) {
      a.expert_token_nums[threadIdx.x] = grand;
      a.ep_send_counts[threadIdx.x] = excl;
    }
  }
  __syncthreads();
  if (rank == 0 && threadIdx.x == 0) {
    a.ep_send_counts[E] = total;
    if (a.dev_status) *a.dev_status = status_all;
  }
  // pair -> slot per token (contiguous per thread); each pair's t * K + k into
  // the block's expert-ordered list for the slot -> pair half. Every pair's
  // rank and base are loaded before any store, so the loads overlap.
#pragma unroll
  for (int i = 0; i < TPT; ++i) {
    const int t = t0 + i * NT + threadIdx.x;
    if (t >= a.bs) continue;
    int slot[KM], pos[KM];
#pragma unroll
    for (int k = 0; k < KM; ++k) {
      slot[k] = -1;
      pos[k] = 0;
      const int ex = e[i][k];
      if (k < a.K && ex >= 0) {
        const int r = cta_rank<NT>(mp, i, S, ex);
        const BaseOfs b = bo[ex];
        slot[k] = b.first + r;
        pos[k] = b.lofs + r;
      }
    }
#pragma unroll
    for (int k = 0; k < KM; ++k) {
      if (k >= a.K || slot[k] < 0) continue;
      ltk[pos[k]] = t * a.K + k;
      if (flat) lex[pos[k]] = static_cast<uint16_t>(e[i][k]);
    }
    store_pair_slots<KM>(a, t, slot);
  }
  __syncthreads();
  if (flat)
    write_flat(a, bo, lex, ltk, listed);
  else
    write_runs(a, &bo[0].first, tot, &bo[0].lofs, ltk, 2);
  for (int s = total + static_cast<int>(rank * blockDim.x + threadIdx.x); s < a.A;
       s += static_cast<int>(cs * blockDim.x))
    a.assist[s] = -1;
  if (!push) {
    __syncwarp();
    cluster_wait_acquire();  // no CTA leaves while another may still read its tot
  }
}

// ---------------------------------------------------------------------------
// Fused dispatch for BS <= 1024 (layout + permute in one launch). Every CTA
// builds the whole layout in shared memory as one CTA of the cluster layout
// would (the ids are at most 64 KB and sit in L2), CTA 0 alone writes the
// layout's outputs, and CTA c copies the rows of tokens [c * per, (c+1) * per)
// to their slots: one thread per 16-byte vector, read once, stored K times.
// NT threads (256 for up to 256 tokens and experts, else 1024). Dynamic shared
// memory: mp[NT / 32][S], bo[E], tot[E].
template <int KM, int NT>
__global__ void __launch_bounds__(NT, 1) dispatch_small_kernel(LayoutArgs a, const uint4* x,
                                                               uint4* expand_x, int V, int per) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int warp_sums[32];
  __shared__ uint32_t status;
  __shared__ int slot_sh[kLayoutSmallMaxTokens / 8][KM];  // slots of this CTA's tokens
  const int E = a.E;
  const int S = cluster_stride(E);
  MaskPre* mp = reinterpret_cast<MaskPre*>(smem);
  BaseOfs* bo = reinterpret_cast<BaseOfs*>(smem + static_cast<size_t>(NT / 32) * S *
                                                      sizeof(MaskPre));
  int* tot = reinterpret_cast<int*>(bo + E);
  const bool writer = blockIdx.x == 0;
  pdl_trigger();
  for (int i = threadIdx.x; i < (NT / 32) * S; i += NT) mp[i] = MaskPre{0u, 0u};
  if (threadIdx.x == 0) status = 0;
  __syncthreads();
  pdl_wait();
  // this CTA's rows are contiguous in x: each thread's first vector is requested
  // now, so its DRAM round trip overlaps the layout work below
  const int t0 = blockIdx.x * per;
  const int t1 = min(a.bs, t0 + per);
  const int nvec = (t1 - t0) * V;
  const uint4* xr = x + static_cast<size_t>(t0) * V;
  uint4 first = make_uint4(0u, 0u, 0u, 0u);
  if (static_cast<int>(threadIdx.x) < nvec) first = ld_nc_v4(xr + threadIdx.x);
  int e[1][KM];
  cta_count_scan<KM, 1, NT>(a, 0, S, mp, tot, &status, e);
  __syncthreads();
  const int cnt = threadIdx.x < E ? tot[threadIdx.x] : 0;
  int total;
  const int excl = block_exclusive_scan(cnt, warp_sums, &total);
  if (threadIdx.x < E) {
    bo[threadIdx.x] = BaseOfs{excl, 0};
    if (writer) {
      a.expert_token_nums[threadIdx.x] = cnt;
      a.ep_send_counts[threadIdx.x] = excl;
    }
  }
  if (writer && threadIdx.x == 0) a.ep_send_counts[E] = total;
  __syncthreads();
  const int t = threadIdx.x;
  if (t < a.bs) {
    int slot[KM];
#pragma unroll
    for (int k = 0; k < KM; ++k)
      slot[k] = (k < a.K && e[0][k] >= 0) ? bo[e[0][k]].first + cta_rank<NT>(mp, 0, S, e[0][k])
                                          : -1;
    if (writer) write_slots<KM>(a, t, slot);
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
  for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
    const int tl = i / V;
    const int v = i - tl * V;
    const uint4 val = i == static_cast<int>(threadIdx.x) ? first : ld_nc_v4(xr + i);
    for (int k = 0; k < a.K; ++k) {
      const int s = slot_sh[tl][k];
      if (s >= 0) st_v4(expand_x + static_cast<size_t>(s) * V + v, val);
    }
  }
}

// ---------------------------------------------------------------------------
// Multi-CTA layout. Workspace: tile_counts[T][E] int32 (turned into their
// exclusive prefix over tiles by the column scan), totals[E], tile_status[T].

struct TileWs {
  int32_t* counts;
  int32_t* totals;
  uint32_t* status;
};

__device__ __forceinline__ TileWs tile_ws(const LayoutArgs& a, int T) {
  TileWs w;
  w.counts = static_cast<int32_t*>(a.workspace);
  w.totals = w.counts + static_cast<size_t>(T) * a.E;
  w.status = reinterpret_cast<uint32_t*>(w.totals + a.E);
  return w;
}

constexpr int kTileWarps = kLayoutTileTokens / 32;

// Phase 1: per-tile expert counts and status bits.
template <int KM>
__global__ void __launch_bounds__(kLayoutTileTokens) layout_count_kernel(LayoutArgs a, int T) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t* words = reinterpret_cast<uint32_t*>(smem);  // [kTileWarps][E]
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

// Phase 2: per expert, the exclusive prefix of the tile counts over tiles (in
// place) and the expert total. A CTA takes 32 experts; its 32 warps split the
// tiles into 32 segments (lane = expert, so each warp reads 32 consecutive
// counts), sum their segment, take the prefix over segments from shared
// memory, and rewrite their segment.
__global__ void __launch_bounds__(1024) layout_colscan_kernel(LayoutArgs a, int T) {
  __shared__ int part[32][33];
  pdl_trigger();
  pdl_wait();
  const int el = threadIdx.x & 31, seg = threadIdx.x >> 5;
  const int ex = blockIdx.x * 32 + el;
  const int per = (T + 31) / 32;
  const int i0 = min(T, seg * per), i1 = min(T, i0 + per);
  const TileWs ws = tile_ws(a, T);
  int sum = 0;
  if (ex < a.E)
    for (int i = i0; i < i1; ++i) sum += ws.counts[static_cast<size_t>(i) * a.E + ex];
  part[seg][el] = sum;
  __syncthreads();
  int run = 0;
  for (int g = 0; g < seg; ++g) run += part[g][el];
  if (ex < a.E) {
    if (seg == 31) ws.totals[ex] = run + sum;
    for (int i = i0; i < i1; ++i) {
      const size_t at = static_cast<size_t>(i) * a.E + ex;
      const int c = ws.counts[at];
      ws.counts[at] = run;
      run += c;
    }
  }
}

// Phase 3 for one 256-token tile, run by a whole CTA: the tile's first slot
// per expert (its prefix over earlier tiles + the exclusive scan of the expert
// totals), then slot[] of this thread's token (t < BS). The CTA with first_cta
// writes the counts, prefix sums and status word. Shared memory (dynamic):
// words[kTileWarps][E], base[E], total[E].
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
  // the workspace loads below
  const int t = tile * kLayoutTileTokens + threadIdx.x;
#pragma unroll
  for (int k = 0; k < KM; ++k) e[k] = -1;
  if (t < a.bs) classify_row<KM>(a, t, e);
  const TileWs ws = tile_ws(a, T);
  for (int ex = threadIdx.x; ex < E; ex += blockDim.x) {
    base[ex] = ws.counts[static_cast<size_t>(tile) * E + ex];
    total[ex] = ws.totals[ex];
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

// Phase 3 as its own launch: every tile's slots (the slot -> pair half written
// run by run, see write_runs), and -1 for the unused slots [R, A). Dynamic
// shared memory: tile_slots' words[kTileWarps][E], base[E], total[E], then
// cnt[E], lofs[E] and ltk[kLayoutTileTokens * K].
template <int KM>
__global__ void __launch_bounds__(kLayoutTileTokens) layout_scatter_kernel(LayoutArgs a, int T) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int warp_sums[32];
  __shared__ uint32_t status;
  pdl_trigger();
  pdl_wait();
  const int E = a.E;
  uint32_t* words = reinterpret_cast<uint32_t*>(smem);
  int* base = reinterpret_cast<int*>(words + kTileWarps * E);
  int* cnt = base + 2 * E;
  int* lofs = cnt + E;
  int* ltk = lofs + E;
  int e[KM], slot[KM], grand;
  tile_slots<KM>(a, T, blockIdx.x, blockIdx.x == 0, words, warp_sums, &status, e, slot, &grand);
  // the tile's own count per expert and their exclusive scan (each thread a run of experts)
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = min(E, static_cast<int>(threadIdx.x) * per), e1 = min(E, e0 + per);
  int run = 0;
  for (int ex = e0; ex < e1; ++ex) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kTileWarps; ++w) c += __popc(words[w * E + ex]);
    cnt[ex] = c;
    run += c;
  }
  int tile_total;
  int off = block_exclusive_scan(run, warp_sums, &tile_total);
  for (int ex = e0; ex < e1; ++ex) {
    lofs[ex] = off;
    off += cnt[ex];
  }
  __syncthreads();
  const int t = blockIdx.x * kLayoutTileTokens + threadIdx.x;
  if (t < a.bs) {
    const size_t A = static_cast<size_t>(a.A);
#pragma unroll
    for (int k = 0; k < KM; ++k) {
      if (k >= a.K) continue;
      const int tk = t * a.K + k;
      if (e[k] >= 0) ltk[lofs[e[k]] + slot[k] - base[e[k]]] = tk;
      a.assist[A + tk] = e[k] >= 0 ? slot[k] : -1;
    }
  }
  __syncthreads();
  write_runs(a, base, cnt, lofs, ltk, 1);
  for (int s = grand + blockIdx.x * blockDim.x + threadIdx.x; s < a.A;
       s += gridDim.x * blockDim.x)
    a.assist[s] = -1;
}

template <int KM, int NT>
cudaError_t launch_dispatch_small_nt(const LayoutArgs& a, const void* x, void* expand_x, int H,
                                     cudaStream_t st) {
  const int V = H / kVecElems;
  // at most kLayoutSmallMaxTokens / 8 tokens per CTA (the slot buffer's size)
  int blocks = sm_count();
  if (blocks > a.bs) blocks = a.bs > 0 ? a.bs : 1;
  int per = (a.bs + blocks - 1) / blocks;
  if (per > kLayoutSmallMaxTokens / 8) per = kLayoutSmallMaxTokens / 8;
  if (per < 1) per = 1;
  blocks = a.bs > 0 ? (a.bs + per - 1) / per : 1;
  const size_t smem = cluster_smem_bytes(a.E, 1, NT);
  cudaError_t err = cudaFuncSetAttribute(dispatch_small_kernel<KM, NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  return launch_pdl(dispatch_small_kernel<KM, NT>, dim3(blocks), dim3(NT), smem, st, a,
                    static_cast<const uint4*>(x), static_cast<uint4*>(expand_x), V, per);
}

template <int KM>
cudaError_t launch_dispatch_small_k(const LayoutArgs& a, const void* x, void* expand_x, int H,
                                    cudaStream_t st) {
  if (a.bs <= 256 && a.E <= 256) return launch_dispatch_small_nt<KM, 256>(a, x, expand_x, H, st);
  return launch_dispatch_small_nt<KM, 1024>(a, x, expand_x, H, st);
}

// The cluster layout: CS <= 16 CTAs of NT threads, one token per thread: 256
// threads for up to 256 tokens and experts (one block), 512 up to 8192 tokens
// and E <= 512, so that up to 16 SMs share the work, else 1024.
#ifndef MOE_LAYOUT_PUSH
#define MOE_LAYOUT_PUSH 1
#endif
#ifndef MOE_LAYOUT_CLUSTER_MAX_TOKENS
#define MOE_LAYOUT_CLUSTER_MAX_TOKENS (16 * 1024)
#endif
constexpr int kClusterMaxTokens = MOE_LAYOUT_CLUSTER_MAX_TOKENS;
constexpr size_t kClusterSmemMax = 210 * 1024;

// The kernel gives each expert one thread (its grand total, scan entry and first
// slot), so E <= threads: 512 threads only for E <= 512.
int cluster_threads(int bs, int E) {
  if (bs <= 256 && E <= 256) return 256;
  return (bs <= 16 * 512 && E <= 512) ? 512 : 1024;
}

// Workspace of the tiled path: tile counts, expert totals, tile status words.
size_t tiled_workspace_bytes(int bs, int E) {
  const size_t T = (static_cast<size_t>(bs) + kLayoutTileTokens - 1) / kLayoutTileTokens;
  return T * static_cast<size_t>(E) * 4 + static_cast<size_t>(E) * 4 + T * 4;
}
int cluster_tpt(int bs) { return 1; }

bool cluster_layout_applies(int bs, int E, int K) {
  const int nt = cluster_threads(bs, E);
  return bs <= kClusterMaxTokens && E <= nt &&
         cluster_kernel_smem_bytes(E, cluster_tpt(bs), K, nt) <= kClusterSmemMax;
}

template <int KM, int TPT, int NT>
cudaError_t launch_layout_cluster(const LayoutArgs& a, cudaStream_t st, bool* fits) {
  constexpr auto kernel = layout_cluster_kernel<KM, TPT, NT>;
  // the flat slot -> pair writer when its expert list fits as well
  const int flat = cluster_kernel_smem_bytes(a.E, TPT, a.K, NT, true) <= kClusterSmemMax ? 1 : 0;
  int cs_launch = (a.bs + TPT * NT - 1) / (TPT * NT);
  if (cs_launch < 1) cs_launch = 1;
  // the pushed exchange when its [cs][E] totals and [cs] status words fit the
  // pair-list area
  const int push = MOE_LAYOUT_PUSH && cs_launch * (a.E + 1) <= TPT * NT * a.K ? 1 : 0;
  const size_t smem = cluster_kernel_smem_bytes(a.E, TPT, a.K, NT, flat != 0);
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  int cs = (a.bs + TPT * NT - 1) / (TPT * NT);
  if (cs < 1) cs = 1;
  if (cs > 8) {  // clusters of more than 8 CTAs are opted into per kernel
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (err != cudaSuccess) return err;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  // a cluster this device cannot hold at all: the tiled path instead (host-side
  // query, before any launch)
  int clusters = 0;
  cfg.numAttrs = 1;
  err = cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg);
  cfg.numAttrs = 2;
  if (err != cudaSuccess || clusters < 1) {
    cudaGetLastError();
    *fits = false;
    return cudaSuccess;
  }
  *fits = true;
  return cudaLaunchKernelEx(&cfg, kernel, a, flat, push);
}

template <int KM>
cudaError_t launch_layout_k(const LayoutArgs& a, cudaStream_t st) {
  if (cluster_layout_applies(a.bs, a.E, a.K)) {
    bool fits = false;
    const int nt = cluster_threads(a.bs, a.E);
    const cudaError_t err = nt == 256   ? launch_layout_cluster<KM, 1, 256>(a, st, &fits)
                            : nt == 512 ? launch_layout_cluster<KM, 1, 512>(a, st, &fits)
                                        : launch_layout_cluster<KM, 1, 1024>(a, st, &fits);
    if (err != cudaSuccess || fits) return err;
    // a device that cannot hold the cluster: the tiled path, if given its workspace
    if (a.workspace == nullptr || a.workspace_bytes < tiled_workspace_bytes(a.bs, a.E))
      return cudaErrorInvalidClusterSize;
  }
  const int T = (a.bs + kLayoutTileTokens - 1) / kLayoutTileTokens;
  const size_t smem_count = static_cast<size_t>(kTileWarps) * a.E * sizeof(uint32_t);
  const size_t smem_scatter = smem_count + 4u * a.E * sizeof(int) +
                              static_cast<size_t>(kLayoutTileTokens) * a.K * sizeof(int);
  cudaError_t err = launch_pdl(layout_count_kernel<KM>, dim3(T), dim3(kLayoutTileTokens),
                               smem_count, st, a, T);
  if (err != cudaSuccess) return err;
  err = launch_pdl(layout_colscan_kernel, dim3((a.E + 31) / 32), dim3(1024), 0, st, a, T);
  if (err != cudaSuccess) return err;
  if (smem_scatter > 48 * 1024) {  // E = 1024 with K = 16: up to 64 KB
    err = cudaFuncSetAttribute(layout_scatter_kernel<KM>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_scatter));
    if (err != cudaSuccess) return err;
  }
  return launch_pdl(layout_scatter_kernel<KM>, dim3(T), dim3(kLayoutTileTokens), smem_scatter,
                    st, a, T);
}

}  // namespace

bool dispatch_small_fits(int E, int K) {
  const size_t stat = static_cast<size_t>(kLayoutSmallMaxTokens / 8) * K * 4 + 1024;
  return cluster_smem_bytes(E, 1) + stat <= kClusterSmemMax;
}

cudaError_t launch_dispatch_small(const LayoutArgs& a, const void* x, void* expand_x, int H,
                                  cudaStream_t st) {
  if (a.K <= 2) return launch_dispatch_small_k<2>(a, x, expand_x, H, st);
  if (a.K <= 4) return launch_dispatch_small_k<4>(a, x, expand_x, H, st);
  if (a.K <= 8) return launch_dispatch_small_k<8>(a, x, expand_x, H, st);
  return launch_dispatch_small_k<16>(a, x, expand_x, H, st);
}

size_t layout_workspace_bytes(int bs, int E, int K) {
  return cluster_layout_applies(bs, E, K) ? 0 : tiled_workspace_bytes(bs, E);
}

cudaError_t launch_layout(const LayoutArgs& a, cudaStream_t st) {
  if (a.K <= 2) return launch_layout_k<2>(a, st);
  if (a.K <= 4) return launch_layout_k<4>(a, st);
  if (a.K <= 8) return launch_layout_k<8>(a, st);
  return launch_layout_k<16>(a, st);
}

}  // namespace moe
