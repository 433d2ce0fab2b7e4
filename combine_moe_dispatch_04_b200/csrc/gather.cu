// Combine forward and dispatch backward with every token's rows staged in
// shared memory by the bulk-copy engine. [combine] Function (Formula; special
// expert use cases), Parameters, Return Value; dispatch backward is the same
// gather with unit weights.
//
// One CTA per SM share (persistent grid), warp-specialised. A unit of work is
// one column chunk of one token's output row. The producer warp loads the pair
// metadata (weight, slot, id, mask) of several tokens at once, one lane per
// pair, a batch ahead of use; per unit it waits until the consumers have
// released the stage buffer ("empty" mbarrier), records the K pairs in shared
// memory and starts one cp.async.bulk (global -> shared) per routed row chunk,
// plus ori_x's chunk for a token with a copy/const pair and shared_expert_x's
// chunk, all completing on the buffer's "full" mbarrier. Eight consumer warps
// wait for "full", accumulate each 16-byte vector in fp32 in ascending k from
// shared memory (products with __fmul_rn, sums rounded on their own: the same
// operations, in the same order, as the one-shot kernel, so the output is bit
// for bit the same), add shared_expert_x once, narrow with round-to-nearest-
// even, store the vector, and release the buffer. The number of bytes in flight
// is set by the stage buffers, not by registers, and the metadata loads never
// sit on the consumers' path.
//
// Every wait is bounded (global timer). A warp whose wait gives up marks the
// CTA aborted and leaves its loop; at the end thread 0 counts the CTA in the
// timeout counter and waits (bounded) for every bulk copy the producer started
// and no consumer saw complete, so no copy is left writing into shared memory
// after the CTA exits. The work of an aborted CTA is left unwritten.
#include "async.cuh"
#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int kGConsumerWarps = 8;
constexpr int kGConsumers = 32 * kGConsumerWarps;
constexpr int kGThreads = kGConsumers + 32;  // the last warp is the producer
constexpr int kGMaxBuf = 8;
constexpr uint32_t kGStageTarget = 32 * 1024;  // bytes of row chunks per stage, at most
constexpr uint32_t kGBufBudget = 96 * 1024;    // bytes of stages per CTA (two CTAs per SM)

enum GKind : int { gSkip = 0, gRouted = 1, gZero = 2, gCopy = 3, gConst = 4 };

struct GMeta {
  int kind;
  int row;  // slot of a routed pair, const-expert row j of a const pair
  float w;
};

struct GPlan {
  int nchunks;    // column chunks per token row
  int cw;         // 16-byte vectors per chunk (the last chunk may be shorter)
  int nbuf;       // stage buffers
  int rows;       // row chunks per stage: KMAX (+1 ori_x) (+1 shared_expert_x)
  uint32_t meta;  // byte offset of the metadata
  uint32_t data;  // byte offset of the stage buffers (128-byte aligned)
  uint32_t smem;  // dynamic shared memory bytes
};

// Shared memory: full[kGMaxBuf], empty[kGMaxBuf] mbarriers, then control words
// (abort flag, units issued, units consumed per consumer warp), then per stage
// KMAX GMeta and one int (the unit needs ori_x), then the stage buffers.
constexpr uint32_t kGFull = 0;
constexpr uint32_t kGEmpty = 8 * kGMaxBuf;
constexpr uint32_t kGCtl = 16 * kGMaxBuf;
constexpr uint32_t kGHeader = kGCtl + 4 * (2 + kGConsumerWarps);

// One pair's raw metadata (every load issued at once, none depends on another).
struct GRaw {
  float w;
  int s;
  int id;
  int act;
};

template <bool SPECIAL, bool UNIT>
__device__ __forceinline__ GRaw g_load(const CombineArgs& a, int t, int k) {
  GRaw r{1.0f, -1, -1, 0};
  if (t < a.bs && k < a.K) {
    const size_t tk = static_cast<size_t>(t) * a.K + k;
    if (!UNIT) r.w = __ldg(a.weights + tk);
    r.s = __ldg(a.assist + static_cast<size_t>(a.A) + tk);
    if (SPECIAL) r.id = __ldg(a.topk_idx + tk);
    r.act = pair_active(a.mask, a.mask_ndim, t, k, a.K) ? 1 : 0;
  }
  return r;
}

// Classifies the pair of this lane (lane = group * KP + k): a masked, invalid or
// repeated id takes no part; zero/copy/const experts by id range; a routed pair
// with a slot reads its row.
template <int KP, bool SPECIAL>
__device__ __forceinline__ GMeta g_classify(const CombineArgs& a, const GRaw& r, int lane) {
  GMeta m{gSkip, 0, r.w};
  if (SPECIAL) {
    const int km = lane % KP;
    bool dup = false;
#pragma unroll
    for (int jj = 0; jj < KP; ++jj) {
      const int other = __shfl_sync(0xFFFFFFFFu, r.id, (lane & ~(KP - 1)) | jj);
      dup |= jj < km && other == r.id;
    }
    if (!r.act || r.id < 0 || r.id >= a.E + a.Z + a.C + a.Q || dup) return m;
    if (r.id >= a.E) {
      m.kind = r.id < a.E + a.Z ? gZero : r.id < a.E + a.Z + a.C ? gCopy : gConst;
      m.row = r.id - (a.E + a.Z + a.C);
      return m;
    }
  }
  if (r.act && r.s >= 0) {
    m.kind = gRouted;
    m.row = r.s;
  }
  return m;
}

template <typename T16, int KMAX, bool SPECIAL, bool UNIT, bool SHARED>
__global__ void __launch_bounds__(kGThreads, 2)
    gather_staged_kernel(CombineArgs a, GPlan p, WaitCfg wc, unsigned* timeouts) {
  constexpr int KP = KMAX;     // producer lanes per token
  constexpr int TB = 32 / KP;  // tokens per metadata batch
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGFull);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + kGEmpty);
  volatile int* ctl = reinterpret_cast<volatile int*>(smem + kGCtl);  // abort, issued, prog[]
  GMeta* meta = reinterpret_cast<GMeta*>(smem + p.meta);
  int* need_ori = reinterpret_cast<int*>(smem + p.meta + p.nbuf * KMAX * sizeof(GMeta));
  uint4* data = reinterpret_cast<uint4*>(smem + p.data);
  const int V = a.H / kVecElems;
  const int K = a.K;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const size_t stage_vecs = static_cast<size_t>(p.rows) * p.cw;
  if (threadIdx.x == 0) {
    for (int b = 0; b < p.nbuf; ++b) {
      mbar_init(full + b, 1);
      mbar_init(empty + b, kGConsumerWarps);
    }
    ctl[0] = 0;
    ctl[1] = 0;
    mbar_init_fence();
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();
  const int stride = gridDim.x;

  if (warp == kGConsumerWarps) {
    // ---- producer
    const uint4* Y = static_cast<const uint4*>(a.expand_x);
    const uint4* ori = static_cast<const uint4*>(a.ori_x);
    const uint4* shr = static_cast<const uint4*>(a.shared);
    const int grp = lane / KP, km = lane % KP;
    const uint32_t gbits = KP == 32 ? 0xFFFFFFFFu : ((1u << KP) - 1u);
    int q = 0;
    bool stop = false;
    GRaw nxt = g_load<SPECIAL, UNIT>(a, blockIdx.x + grp * stride, km);
    for (int j0 = 0; !stop && blockIdx.x + j0 * stride < a.bs; j0 += TB) {
      const GRaw cur = nxt;  // the next batch's loads go out before this one is used
      nxt = g_load<SPECIAL, UNIT>(a, blockIdx.x + (j0 + TB + grp) * stride, km);
      const GMeta pm = g_classify<KP, SPECIAL>(a, cur, lane);
      const uint32_t routed = __ballot_sync(0xFFFFFFFFu, pm.kind == gRouted);
      const uint32_t oris =
          SPECIAL ? __ballot_sync(0xFFFFFFFFu, pm.kind == gCopy || pm.kind == gConst) : 0u;
      for (int j = 0; j < TB && !stop; ++j) {
        const int t = blockIdx.x + (j0 + j) * stride;
        if (t >= a.bs) break;
        const uint32_t gm = gbits << (j * KP);
        const int nrouted = __popc(routed & gm);
        const bool with_ori = SPECIAL && (oris & gm) != 0u;
        for (int c = 0; c < p.nchunks; ++c, ++q) {
          const int b = q % p.nbuf;
          if (q >= p.nbuf) {  // wait until every consumer warp has released buffer b
            const bool ok = mbar_wait_bounded(empty + b, ((q / p.nbuf) - 1) & 1, wc.limit_ns);
            if (!__all_sync(0xFFFFFFFFu, ok)) {
              if (lane == 0) ctl[0] = 1;
              stop = true;
              break;
            }
          }
          if (grp == j) meta[b * KMAX + km] = pm;
          if (lane == 0) need_ori[b] = with_ori ? 1 : 0;
          fence_proxy_async_smem();  // the buffer was last read by the consumers' loads
          const int v0 = c * p.cw;
          const int len = min(p.cw, V - v0);
          const uint32_t cb = static_cast<uint32_t>(len) * 16u;
          const uint32_t n = static_cast<uint32_t>(nrouted + (with_ori ? 1 : 0) + (SHARED ? 1 : 0));
          if (wc.withhold == q && blockIdx.x == 0) {  // test hook: 16 bytes that never come
            if (lane == 0) mbar_arrive_expect_tx(full + b, 16u);
            continue;
          }
          if (lane == 0) mbar_arrive_expect_tx(full + b, n * cb);
          __syncwarp();
          uint4* st = data + static_cast<size_t>(b) * stage_vecs;
          if (grp == j && pm.kind == gRouted)
            bulk_g2s(st + static_cast<size_t>(km) * p.cw, Y + static_cast<size_t>(pm.row) * V + v0,
                     cb, full + b);
          if (lane == 0) {
            if (with_ori)
              bulk_g2s(st + static_cast<size_t>(KMAX) * p.cw, ori + static_cast<size_t>(t) * V + v0,
                       cb, full + b);
            if (SHARED)
              bulk_g2s(st + static_cast<size_t>(KMAX + (SPECIAL ? 1 : 0)) * p.cw,
                       shr + static_cast<size_t>(t) * V + v0, cb, full + b);
          }
        }
      }
    }
    if (lane == 0) ctl[1] = q;
  } else {
    // ---- consumers
    uint4* out = static_cast<uint4*>(a.out);
    int q = 0;
    bool stop = false;
    for (int t = blockIdx.x; t < a.bs && !stop; t += stride) {
      for (int c = 0; c < p.nchunks; ++c, ++q) {
        const int b = q % p.nbuf;
        const bool ok = mbar_wait_bounded(full + b, (q / p.nbuf) & 1, wc.limit_ns);
        if (!__all_sync(0xFFFFFFFFu, ok)) {
          if (lane == 0) ctl[0] = 1;
          stop = true;
          break;
        }
        const GMeta* pm = meta + b * KMAX;
        const uint4* st = data + static_cast<size_t>(b) * stage_vecs;
        const bool with_ori = SPECIAL && need_ori[b] != 0;
        const int v0 = c * p.cw;
        const int len = min(p.cw, V - v0);
        for (int v = threadIdx.x; v < len; v += kGConsumers) {
          float acc[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
          float orf[8];
          if (with_ori) widen8<T16>(st[static_cast<size_t>(KMAX) * p.cw + v], orf);
#pragma unroll
          for (int k = 0; k < KMAX; ++k) {
            if (k >= K) break;
            const GMeta m = pm[k];
            if (m.kind == gSkip) continue;
            float val[8];
            if (!SPECIAL || m.kind == gRouted) {
              widen8<T16>(st[static_cast<size_t>(k) * p.cw + v], val);
            } else if (m.kind == gZero) {
#pragma unroll
              for (int i = 0; i < 8; ++i) val[i] = 0.0f;
            } else if (m.kind == gCopy) {
#pragma unroll
              for (int i = 0; i < 8; ++i) val[i] = orf[i];
            } else {  // alpha_1 * ori_x + alpha_2 * v, each product and the sum rounded
              const size_t r = static_cast<size_t>(m.row) * V + v0 + v;
              float a1[8], a2[8], cv[8];
              widen8<T16>(__ldg(static_cast<const uint4*>(a.alpha1) + r), a1);
              widen8<T16>(__ldg(static_cast<const uint4*>(a.alpha2) + r), a2);
              widen8<T16>(__ldg(static_cast<const uint4*>(a.const_v) + r), cv);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                val[i] = __fadd_rn(__fmul_rn(a1[i], orf[i]), __fmul_rn(a2[i], cv[i]));
            }
            if (UNIT)
              add8_rn(acc, val);
            else
              axpy8_rn(acc, m.w, val);
          }
          if (SHARED) {
            float sh[8];
            widen8<T16>(st[static_cast<size_t>(KMAX + (SPECIAL ? 1 : 0)) * p.cw + v], sh);
            add8_rn(acc, sh);
          }
          st_v4(out + static_cast<size_t>(t) * V + v0 + v, narrow8<T16>(acc));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + b);  // this warp is done with buffer b
      }
    }
    if (lane == 0) ctl[2 + warp] = q;
  }
  __syncthreads();
  if (threadIdx.x == 0 && ctl[0] != 0) {
    atomicAdd(timeouts, 1u);
    const int issued = ctl[1];
    int lo = issued;
    for (int w = 0; w < kGConsumerWarps; ++w) lo = min(lo, static_cast<int>(ctl[2 + w]));
    for (int u = lo; u < issued; ++u)  // copies started and not seen complete: let them land
      if (!(u == wc.withhold && blockIdx.x == 0)) mbar_wait_bounded(full + u % p.nbuf, (u / p.nbuf) & 1);
  }
}

template <int KMAX>
GPlan g_plan(const CombineArgs& a, bool special, bool shared) {
  GPlan p;
  const int V = a.H / kVecElems;
  p.rows = KMAX + (special ? 1 : 0) + (shared ? 1 : 0);
  const int cw_max = static_cast<int>(kGStageTarget / (static_cast<uint32_t>(p.rows) * 16u));
  p.nchunks = (V + cw_max - 1) / cw_max;
  p.cw = (V + p.nchunks - 1) / p.nchunks;
  const uint32_t stage = static_cast<uint32_t>(p.rows) * p.cw * 16u;
  int nbuf = static_cast<int>(kGBufBudget / stage);
  p.nbuf = nbuf < 2 ? 2 : nbuf > kGMaxBuf ? kGMaxBuf : nbuf;
  p.meta = (kGHeader + 15u) / 16u * 16u;
  const uint32_t meta_end = p.meta + p.nbuf * (KMAX * sizeof(GMeta) + sizeof(int));
  p.data = (meta_end + 127u) / 128u * 128u;
  p.smem = p.data + p.nbuf * stage;
  return p;
}

template <typename T16, int KMAX, bool SPECIAL, bool UNIT, bool SHARED>
cudaError_t g_launch(const CombineArgs& a, const WaitCfg& wc, cudaStream_t st) {
  constexpr auto kernel = gather_staged_kernel<T16, KMAX, SPECIAL, UNIT, SHARED>;
  const GPlan p = g_plan<KMAX>(a, SPECIAL, SHARED);
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(p.smem));
  if (err != cudaSuccess) return err;
  unsigned* timeouts = wait_timeout_counter();
  if (timeouts == nullptr) return cudaErrorInvalidSymbol;
  int per_sm = 0;  // depends on the plan's shared memory: not cached
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kGThreads, p.smem);
  if (err != cudaSuccess) return err;
  const int cap = sm_count() * (per_sm > 0 ? per_sm : 1);
  const int blocks = a.bs < cap ? a.bs : cap;
  return launch_pdl(kernel, dim3(blocks), dim3(kGThreads), p.smem, st, a, p, wc, timeouts);
}

template <typename T16, int KMAX, bool SPECIAL, bool UNIT>
cudaError_t g_launch_s(const CombineArgs& a, const WaitCfg& wc, cudaStream_t st) {
  if (!UNIT && a.shared != nullptr) return g_launch<T16, KMAX, SPECIAL, UNIT, true>(a, wc, st);
  return g_launch<T16, KMAX, SPECIAL, UNIT, false>(a, wc, st);
}

template <typename T16, bool SPECIAL, bool UNIT>
cudaError_t g_launch_k(const CombineArgs& a, const WaitCfg& wc, cudaStream_t st) {
  if (a.K <= 2) return g_launch_s<T16, 2, SPECIAL, UNIT>(a, wc, st);
  if (a.K <= 4) return g_launch_s<T16, 4, SPECIAL, UNIT>(a, wc, st);
  if (a.K <= 8) return g_launch_s<T16, 8, SPECIAL, UNIT>(a, wc, st);
  return g_launch_s<T16, 16, SPECIAL, UNIT>(a, wc, st);
}

template <typename T16>
cudaError_t g_launch_t(const CombineArgs& a, const WaitCfg& wc, cudaStream_t st) {
  if (a.weights == nullptr) return g_launch_k<T16, false, true>(a, wc, st);
  if (a.Z + a.C + a.Q > 0) return g_launch_k<T16, true, false>(a, wc, st);
  return g_launch_k<T16, false, false>(a, wc, st);
}

}  // namespace

bool gather_staged_applies(const CombineArgs& a) {
  return a.bs > 0 && a.H / kVecElems >= kGatherStagedMinVecs;
}

cudaError_t launch_gather_staged(const CombineArgs& a, cudaStream_t st, const WaitCfg& wc) {
  return a.dtype == MOE_BF16 ? g_launch_t<Bf16>(a, wc, st) : g_launch_t<Fp16>(a, wc, st);
}

}  // namespace moe
