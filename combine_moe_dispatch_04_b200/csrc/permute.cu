// Dispatch permute: expand_x[slot(t, k)] = x[t] for every pair with a slot,
// optionally quantised to int8 per token ([combine] Parameters:
// comm_quant_mode 2; Example: quant_mode = 2).
//
// Plain copy: one thread per 16-byte vector of x (coalesced along the row),
// read once and stored to each of the token's K slots; one-shot blocks.
//
// int8: one CTA per token (grid-stride); each thread keeps 16-element chunks
// of the row in registers, the CTA reduces max|x|, and every chunk becomes one
// 16-byte int8 store per slot. With smooth scales (E, H) every slot has its
// own row x[t] * smooth[e] and is quantised on its own, one warp per slot.
#include "async.cuh"
#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int kCopyThreads = 256;
constexpr int kCopyItems = 2;  // vectors per thread, a block apart (1 or 4: no better)

// One thread per 16-byte vector of x (coalesced along the row) in one-shot
// blocks: the vector is read once and stored to each of the token's K slots.
template <int KM>
__global__ void __launch_bounds__(kCopyThreads) permute_copy_kernel(
    const uint4* __restrict__ x, const int32_t* __restrict__ assist, uint4* __restrict__ out,
    int bs, int K, int V, int A) {
  pdl_trigger();
  pdl_wait();
  const int n = bs * V;
  const int32_t* slots_all = assist + static_cast<size_t>(A);
  // a token's K slots are loaded together (16-byte loads when K and A allow),
  // then its K stores go out back to back
  const bool vec4 = KM >= 4 && (K & 3) == 0 && (A & 3) == 0 &&
                    (reinterpret_cast<uintptr_t>(assist) & 15) == 0;
  // every item's vector and slots are requested before any store
  uint4 val[kCopyItems];
  int s[kCopyItems][KM], v[kCopyItems];
#pragma unroll
  for (int i = 0; i < kCopyItems; ++i) {
    const int item = (blockIdx.x * kCopyItems + i) * kCopyThreads + threadIdx.x;
#pragma unroll
    for (int k = 0; k < KM; ++k) s[i][k] = -1;
    v[i] = 0;
    if (item >= n) continue;
    const int t = item / V;
    v[i] = item - t * V;
    val[i] = ld_nc_v4(x + item);
    const int32_t* slots = slots_all + static_cast<size_t>(t) * K;
    if (vec4) {
#pragma unroll
      for (int q = 0; q < KM / 4; ++q) {
        int4 w = make_int4(-1, -1, -1, -1);
        if (4 * q < K) w = __ldg(reinterpret_cast<const int4*>(slots) + q);
        s[i][4 * q] = w.x;
        s[i][4 * q + 1] = w.y;
        s[i][4 * q + 2] = w.z;
        s[i][4 * q + 3] = w.w;
      }
    } else {
#pragma unroll
      for (int k = 0; k < KM; ++k) s[i][k] = k < K ? __ldg(slots + k) : -1;
    }
  }
#pragma unroll
  for (int i = 0; i < kCopyItems; ++i)
#pragma unroll
    for (int k = 0; k < KM; ++k)
      if (s[i][k] >= 0) st_v4(out + static_cast<size_t>(s[i][k]) * V + v[i], val[i]);
}

// CPT 16-element chunks per thread (1, 2 or 4), chosen by the launcher so a
// row fits the CTA with as few registers as possible.
template <typename T16, int CPT>
__global__ void __launch_bounds__(256) permute_quant_kernel(
    const uint4* __restrict__ x, const int32_t* __restrict__ assist, uint4* __restrict__ out,
    float* __restrict__ scales, int bs, int K, int H, int A) {
  // per-warp maxima, two sets used alternately: a warp writes set p for the next
  // token only after that token's barrier, which every warp reaches after
  // reading this token's set, so one barrier per token suffices
  __shared__ float warp_max[2][8];
  int par = 0;
  pdl_trigger();
  pdl_wait();
  const int C = H / 16;  // chunks per row
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  // the CTA's next token row is requested while the current one is quantised
  // and stored (raw 16-bit values, two 16-byte vectors per chunk)
  uint4 next[CPT][2];
  auto load_row = [&](int t) {
    const uint4* xr = x + static_cast<size_t>(t) * (H / 8);
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int c = threadIdx.x + j * blockDim.x;
      if (c < C) {
        next[j][0] = ld_nc_v4(xr + 2 * c);
        next[j][1] = ld_nc_v4(xr + 2 * c + 1);
      }
    }
  };
  if (blockIdx.x < bs) load_row(blockIdx.x);
  for (int t = blockIdx.x; t < bs; t += gridDim.x) {
    uint4 cur[CPT][2];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      cur[j][0] = next[j][0];
      cur[j][1] = next[j][1];
    }
    if (t + static_cast<int>(gridDim.x) < bs) load_row(t + gridDim.x);
    const int32_t* slots = assist + static_cast<size_t>(A) + static_cast<size_t>(t) * K;
    const int my_slot = lane < K ? __ldg(slots + lane) : -1;  // every warp holds the K slots
    float f[CPT][16];
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int c = threadIdx.x + j * blockDim.x;
      if (c < C) {
        float lo[8], hi[8];
        widen8<T16>(cur[j][0], lo);
        widen8<T16>(cur[j][1], hi);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          f[j][i] = lo[i];
          f[j][8 + i] = hi[i];
          amax = fmaxf(amax, fmaxf(fabsf(lo[i]), fabsf(hi[i])));
        }
      }
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, d));
    if (lane == 0) warp_max[par][warp] = amax;
    __syncthreads();
    amax = warp_max[par][0];
    for (int w = 1; w < nwarps; ++w) amax = fmaxf(amax, warp_max[par][w]);
    par ^= 1;
    const float scale = __fdiv_rn(amax, 127.0f);
    const float inv_scale = 1.0f / scale;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int c = threadIdx.x + j * blockDim.x;
      const bool mine = c < C;  // every lane still takes part in the shuffles below
      const uint4 val = mine ? pack_codes16(f[j], amax, scale, inv_scale) : make_uint4(0, 0, 0, 0);
      for (int k = 0; k < K; ++k) {
        const int s = __shfl_sync(0xFFFFFFFFu, my_slot, k);
        if (mine && s >= 0) st_v4(out + static_cast<size_t>(s) * C + c, val);
      }
    }
    if (warp == 0 && lane < K && my_slot >= 0) scales[my_slot] = scale;
  }
}

// Smooth-scaled int8 (reading R18): the row of slot s is y = x[t] * smooth[e]
// for its pair (t, k) and expert e, quantised on its own. One warp per slot,
// slots taken in order (a contiguous run per warp), so the warps of an SM keep
// re-reading one expert's smooth row from L1 and write their int8 rows back to
// back; each token row is gathered K times, from L2 after its first touch.
// Lane i loads the pair and expert of slot i of each batch of 32 and the warp
// walks the batch by shuffle, so only the first slot of a batch waits on the
// index loads. max|y| is a warp reduction: no barriers. With CPL > 0 a lane
// keeps its CPL chunks of y in registers (C <= 32 * CPL); with CPL == 0 it
// streams the row twice, the second pass served mostly by L1.
template <typename T16>
__device__ __forceinline__ void smooth_chunk(const uint4* xr, const float4* sr, int c,
                                             float (&y)[16]) {
  float v[16];
  widen8<T16>(__ldg(xr + 2 * c), reinterpret_cast<float(&)[8]>(v[0]));
  widen8<T16>(__ldg(xr + 2 * c + 1), reinterpret_cast<float(&)[8]>(v[8]));
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 m = __ldg(sr + 4 * c + q);
    y[4 * q + 0] = __fmul_rn(v[4 * q + 0], m.x);
    y[4 * q + 1] = __fmul_rn(v[4 * q + 1], m.y);
    y[4 * q + 2] = __fmul_rn(v[4 * q + 2], m.z);
    y[4 * q + 3] = __fmul_rn(v[4 * q + 3], m.w);
  }
}

constexpr int kSmoothThreads = 256;
constexpr int kSmoothStream = 4;  // chunks per lane in flight when streaming

template <typename T16, int CPL>
__global__ void __launch_bounds__(kSmoothThreads) permute_quant_smooth_kernel(
    const uint4* __restrict__ x, const int32_t* __restrict__ topk_idx,
    const float4* __restrict__ smooth, const int32_t* __restrict__ assist,
    const int32_t* __restrict__ send, uint4* __restrict__ out, float* __restrict__ scales, int K,
    int H, int A, int E) {
  pdl_trigger();
  pdl_wait();
  const int C = H / 16;
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * (kSmoothThreads / 32);
  const int gw = blockIdx.x * (kSmoothThreads / 32) + (threadIdx.x >> 5);
  const int R = min(max(__ldg(send + E), 0), A);
  const int per = (R + nwarps - 1) / nwarps;
  const int lo = gw * per;
  const int hi = min(R, lo + per);
  for (int b = lo; b < hi; b += 32) {
    int my_pair = -1, my_e = -1;
    if (b + lane < hi) {
      my_pair = __ldg(assist + b + lane);
      if (my_pair >= 0) my_e = __ldg(topk_idx + my_pair);
    }
    const int n = min(32, hi - b);
    for (int j = 0; j < n; ++j) {
      const int pair = __shfl_sync(0xFFFFFFFFu, my_pair, j);
      const int e = __shfl_sync(0xFFFFFFFFu, my_e, j);
      if (pair < 0 || static_cast<unsigned>(e) >= static_cast<unsigned>(E)) continue;
      const int s = b + j;
      const uint4* xr = x + static_cast<size_t>(pair / K) * (H / 8);
      const float4* sr = smooth + static_cast<size_t>(e) * (H / 4);
      uint4* orow = out + static_cast<size_t>(s) * C;
      float amax = 0.0f;
      if constexpr (CPL > 0) {
        float y[CPL][16];
#pragma unroll
        for (int u = 0; u < CPL; ++u) {
          const int c = lane + 32 * u;
          if (c < C) {
            smooth_chunk<T16>(xr, sr, c, y[u]);
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(y[u][i]));
          }
        }
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, d));
        const float scale = __fdiv_rn(amax, 127.0f);
        const float inv_scale = 1.0f / scale;
#pragma unroll
        for (int u = 0; u < CPL; ++u) {
          const int c = lane + 32 * u;
          if (c < C) st_v4(orow + c, pack_codes16(y[u], amax, scale, inv_scale));
        }
        if (lane == 0) scales[s] = scale;
      } else {
        for (int c0 = lane; c0 < C; c0 += 32 * kSmoothStream) {
#pragma unroll
          for (int u = 0; u < kSmoothStream; ++u) {
            const int c = c0 + 32 * u;
            if (c < C) {
              float y[16];
              smooth_chunk<T16>(xr, sr, c, y);
#pragma unroll
              for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(y[i]));
            }
          }
        }
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, d));
        const float scale = __fdiv_rn(amax, 127.0f);
        const float inv_scale = 1.0f / scale;
        for (int c0 = lane; c0 < C; c0 += 32 * kSmoothStream) {
#pragma unroll
          for (int u = 0; u < kSmoothStream; ++u) {
            const int c = c0 + 32 * u;
            if (c < C) {
              float y[16];
              smooth_chunk<T16>(xr, sr, c, y);
              st_v4(orow + c, pack_codes16(y, amax, scale, inv_scale));
            }
          }
        }
        if (lane == 0) scales[s] = scale;
      }
    }
  }
}

// Smooth-scaled int8 with each warp's token rows staged in shared memory: a
// CTA takes a contiguous run of slots and its warps take them in turn (so
// they share the current expert's smooth row through L1). The warp loads the
// pairs and experts of 32 of its slots at once; lane 0 starts one bulk copy of
// the token row of the slot kSmoothStages - 1 places ahead into the warp's next buffer
// (cp.async.bulk on the buffer's mbarrier), so the gather is in flight while
// the current slot is quantised. Lane l handles 16-byte vectors l, l + 32, ...
// of the row: one pass for max|x * s| (warp reduction), one for the codes
// (8 bytes per vector). No CTA barrier; every wait is bounded and a warp that
// gives up counts itself in *timeouts and returns.
constexpr int kSmoothStages = 3;

// y[i] = fl(y[i] * s[i]) for eight values, in pairs. y only feeds other
// products and a max, never a sum, so the packed multiply keeps every
// product's own rounding.
__device__ __forceinline__ void smooth_mul8(float (&y)[8], const float4& m0, const float4& m1) {
  const float2 p0 = __fmul2_rn(f2(y[0], y[1]), f2(m0.x, m0.y));
  const float2 p1 = __fmul2_rn(f2(y[2], y[3]), f2(m0.z, m0.w));
  const float2 p2 = __fmul2_rn(f2(y[4], y[5]), f2(m1.x, m1.y));
  const float2 p3 = __fmul2_rn(f2(y[6], y[7]), f2(m1.z, m1.w));
  y[0] = p0.x; y[1] = p0.y; y[2] = p1.x; y[3] = p1.y;
  y[4] = p2.x; y[5] = p2.y; y[6] = p3.x; y[7] = p3.y;
}

struct SmoothSlot {
  int e;     // expert of the slot, -1: nothing to do
  int slot;
};

__host__ __device__ constexpr size_t smooth_warp_bytes(int H) {
  return (128 + static_cast<size_t>(kSmoothStages) * H * 2 + 127) / 128 * 128;
}

// SPL > 0 (H = 256 * SPL): the warp keeps the current expert's smooth row in
// registers (lane l: vectors l, l + 32, ...), reloading it only when the
// expert of its next slot differs, so the per-value smooth factors come from
// registers instead of L1 (whose bandwidth bounded the SPL = 0 form, which
// reads them from L1 in both passes).
// Threads and resident blocks per SM of the staged smooth kernel: with the
// smooth row of H = 2048 in registers a warp needs about 160 of them, so 12
// warps make one block per SM; otherwise 8 warps and two blocks.
template <int SPL>
__host__ __device__ constexpr int smooth_threads() { return SPL >= 8 ? 384 : 256; }
template <int SPL>
__host__ __device__ constexpr int smooth_blocks_per_sm() { return SPL >= 8 ? 1 : 2; }

template <typename T16, int SPL>
__global__ void __launch_bounds__(smooth_threads<SPL>(), smooth_blocks_per_sm<SPL>())
    permute_smooth_staged_kernel(
    const uint4* __restrict__ x, const int32_t* __restrict__ topk_idx,
    const float4* __restrict__ smooth, const int32_t* __restrict__ assist,
    const int32_t* __restrict__ send, uint2* __restrict__ out, float* __restrict__ scales, int K,
    int H, int A, int E, WaitCfg wc, unsigned* timeouts) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int V = H / kVecElems;
  const uint32_t row_bytes = static_cast<uint32_t>(H) * 2u;
  unsigned char* wbase = smem + static_cast<size_t>(warp) * smooth_warp_bytes(H);
  uint64_t* bars = reinterpret_cast<uint64_t*>(wbase);
  SmoothSlot* info = reinterpret_cast<SmoothSlot*>(wbase + 64);
  uint4* rows = reinterpret_cast<uint4*>(wbase + 128);
  if (lane == 0) {
    for (int b = 0; b < kSmoothStages; ++b) mbar_init(bars + b, 1);
    mbar_init_fence();
  }
  __syncwarp();
  pdl_trigger();
  pdl_wait();
  const int R = min(max(__ldg(send + E), 0), A);
  const int per = (R + gridDim.x - 1) / gridDim.x;
  const int lo = blockIdx.x * per;
  const int hi = min(R, lo + per);

  // The warp's q-th slot is lo + warp + q * nwarps. Lane l holds the pair and
  // expert of slot qb + l of the current batch of 32, loaded together, so the
  // index round trips are paid once per 32 slots.
  int qb = -32, my_pair = -1, my_e = -1;
  // test hook: the first warp's slot number wc.withhold waits for bytes that never come
  const int held = (blockIdx.x == 0 && warp == 0) ? wc.withhold : -1;
  // All lanes: slot q into buffer b (lane 0 records it and starts the copy).
  auto stage = [&](int q, int b) {
    if (q >= qb + 32) {
      qb = q;
      const int s = lo + warp + (qb + lane) * nwarps;
      my_pair = s < hi ? __ldg(assist + s) : -1;
      my_e = my_pair >= 0 ? __ldg(topk_idx + my_pair) : -1;
      if (static_cast<unsigned>(my_e) >= static_cast<unsigned>(E)) my_e = -1;
    }
    const int pair = __shfl_sync(0xFFFFFFFFu, my_pair, q - qb);
    const int e = __shfl_sync(0xFFFFFFFFu, my_e, q - qb);
    if (lane == 0) {
      info[b] = SmoothSlot{e, lo + warp + q * nwarps};
      fence_proxy_async_smem();  // the buffer was last read by the warp's loads
      if (q == held) {  // test hook: 16 bytes that never come
        mbar_arrive_expect_tx(bars + b, 16u);
        return;
      }
      mbar_arrive_expect_tx(bars + b, e >= 0 ? row_bytes : 0u);
      if (e >= 0)
        bulk_g2s(rows + static_cast<size_t>(b) * V, x + static_cast<size_t>(pair / K) * V,
                 row_bytes, bars + b);
    }
  };

  for (int p = 0; p < kSmoothStages - 1; ++p)
    if (lo + warp + p * nwarps < hi) stage(p, p);
  float4 sreg[SPL > 0 ? SPL : 1][2];  // the current expert's smooth factors (SPL > 0)
  int cur_e = -1;
  int it = 0;
  for (int s = lo + warp; s < hi; s += nwarps, ++it) {
    const int b = it % kSmoothStages;
    const bool ok = mbar_wait_bounded(bars + b, (it / kSmoothStages) & 1, wc.limit_ns);
    if (__any_sync(0xFFFFFFFFu, !ok)) {
      if (lane == 0) {
        atomicAdd(timeouts, 1u);
        for (int q = 1; q < kSmoothStages; ++q)  // copies already started: let them land
          if (s + q * nwarps < hi && it + q != held)
            mbar_wait_bounded(bars + (it + q) % kSmoothStages, ((it + q) / kSmoothStages) & 1);
      }
      return;
    }
    // the buffer of the previous slot is free (its reads ended before the
    // __syncwarp below): refill it with the slot kSmoothStages - 1 ahead
    if (s + (kSmoothStages - 1) * nwarps < hi)
      stage(it + kSmoothStages - 1, (it + kSmoothStages - 1) % kSmoothStages);
    const SmoothSlot si = info[b];
    if constexpr (SPL > 0) {
      if (si.e >= 0) {
        if (si.e != cur_e) {  // warp-uniform: the slot's expert is in shared memory
          const float4* sr = smooth + static_cast<size_t>(si.e) * (H / 4);
#pragma unroll
          for (int j = 0; j < SPL; ++j) {
            const int v = lane + 32 * j;
            sreg[j][0] = __ldg(sr + 2 * v);
            sreg[j][1] = __ldg(sr + 2 * v + 1);
          }
          cur_e = si.e;
        }
        const uint4* xr = rows + static_cast<size_t>(b) * V;
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < SPL; ++j) {
          float y[8];
          widen8<T16>(xr[lane + 32 * j], y);
          smooth_mul8(y, sreg[j][0], sreg[j][1]);
          amax = fmaxf(amax, absmax8(y));
        }
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, d));
        const float scale = __fdiv_rn(amax, 127.0f);
        const float inv_scale = 1.0f / scale;
        uint2* orow = out + static_cast<size_t>(si.slot) * V;
#pragma unroll
        for (int j = 0; j < SPL; ++j) {
          float y[8];
          widen8<T16>(xr[lane + 32 * j], y);
          smooth_mul8(y, sreg[j][0], sreg[j][1]);
          orow[lane + 32 * j] = pack_codes8(y, amax, scale, inv_scale);
        }
        if (lane == 0) scales[si.slot] = scale;
      }
      __syncwarp();
      continue;
    }
    if (si.e >= 0) {
      const uint4* xr = rows + static_cast<size_t>(b) * V;
      const float4* sr = smooth + static_cast<size_t>(si.e) * (H / 4);
      float amax = 0.0f;
#pragma unroll 4
      for (int v = lane; v < V; v += 32) {
        float y[8];
        widen8<T16>(xr[v], y);
        const float4 m0 = __ldg(sr + 2 * v), m1 = __ldg(sr + 2 * v + 1);
        smooth_mul8(y, m0, m1);
        amax = fmaxf(amax, absmax8(y));
      }
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, d));
      const float scale = __fdiv_rn(amax, 127.0f);
      const float inv_scale = 1.0f / scale;
      uint2* orow = out + static_cast<size_t>(si.slot) * V;
#pragma unroll 4
      for (int v = lane; v < V; v += 32) {
        float y[8];
        widen8<T16>(xr[v], y);
        const float4 m0 = __ldg(sr + 2 * v), m1 = __ldg(sr + 2 * v + 1);
        smooth_mul8(y, m0, m1);
        orow[v] = pack_codes8(y, amax, scale, inv_scale);
      }
      if (lane == 0) scales[si.slot] = scale;
    }
    __syncwarp();
  }
}

// Threads and 16-element chunks per thread for the int8 kernels: one chunk
// per thread up to 256 threads, then 2 or 4 (H <= 16384, checked by the caller).
void quant_shape(int H, int* threads, int* cpt) {
  const int C = H / 16;
  int t = (C + 31) / 32 * 32;
  t = t > 256 ? 256 : t;
  *threads = t;
  *cpt = (C + t - 1) / t;
}

}  // namespace

cudaError_t launch_permute_smooth(const PermuteArgs& a, const int32_t* topk_idx,
                                  const float* smooth, const int32_t* send, int E,
                                  cudaStream_t st, const WaitCfg& wc, bool staged_only) {
  if (a.bs == 0 || a.A == 0) return cudaSuccess;
  const int C = a.H / 16;
  const bool bf = a.dtype == MOE_BF16;
  auto kern = bf ? permute_quant_smooth_kernel<Bf16, 0> : permute_quant_smooth_kernel<Fp16, 0>;
  if (C <= 32)
    kern = bf ? permute_quant_smooth_kernel<Bf16, 1> : permute_quant_smooth_kernel<Fp16, 1>;
  else if (C <= 64)
    kern = bf ? permute_quant_smooth_kernel<Bf16, 2> : permute_quant_smooth_kernel<Fp16, 2>;
  else if (C <= 128)
    kern = bf ? permute_quant_smooth_kernel<Bf16, 4> : permute_quant_smooth_kernel<Fp16, 4>;
  // Staged kernel when at least four warps' buffers fit in 110 KB (two CTAs per SM).
  const int staged_warps = static_cast<int>(110 * 1024 / smooth_warp_bytes(a.H));
  if (staged_warps >= 4) {
    int warps = staged_warps < 8 ? staged_warps : 8;
    auto sk = bf ? permute_smooth_staged_kernel<Bf16, 0> : permute_smooth_staged_kernel<Fp16, 0>;
    if (a.H % 256 == 0 && a.H <= 2048) {  // the smooth row fits in a warp's registers
      const int spl = a.H / 256;
      if (spl == 1) sk = bf ? permute_smooth_staged_kernel<Bf16, 1> : permute_smooth_staged_kernel<Fp16, 1>;
      if (spl == 2) sk = bf ? permute_smooth_staged_kernel<Bf16, 2> : permute_smooth_staged_kernel<Fp16, 2>;
      if (spl == 4) sk = bf ? permute_smooth_staged_kernel<Bf16, 4> : permute_smooth_staged_kernel<Fp16, 4>;
      if (spl == 8) {  // one block of 12 warps per SM (smooth_threads<8>)
        sk = bf ? permute_smooth_staged_kernel<Bf16, 8> : permute_smooth_staged_kernel<Fp16, 8>;
        warps = smooth_threads<8>() / 32;
      }
    }
    const size_t smem = static_cast<size_t>(warps) * smooth_warp_bytes(a.H);
    cudaError_t err = cudaFuncSetAttribute(sk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    unsigned* timeouts = wait_timeout_counter();
    if (timeouts == nullptr) return cudaErrorInvalidSymbol;
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sk, 32 * warps, smem);
    if (err != cudaSuccess) return err;
    const long long want = (static_cast<long long>(a.A) + warps - 1) / warps;
    const long long cap = static_cast<long long>(sm_count()) * (per_sm > 0 ? per_sm : 1);
    const int blocks = static_cast<int>(want < cap ? want : cap);
    return launch_pdl(sk, dim3(blocks), dim3(32 * warps), smem, st,
                      static_cast<const uint4*>(a.x), topk_idx,
                      reinterpret_cast<const float4*>(smooth), a.assist, send,
                      static_cast<uint2*>(a.expand_x), a.scales, a.K, a.H, a.A, E, wc,
                      timeouts);
  }
  if (staged_only) return cudaErrorNotSupported;
  int per_sm = 0;
  cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kSmoothThreads, 0);
  if (err != cudaSuccess) return err;
  const long long want = (static_cast<long long>(a.A) + kSmoothThreads / 32 - 1) /
                         (kSmoothThreads / 32);
  const long long cap = static_cast<long long>(sm_count()) * (per_sm > 0 ? per_sm : 1);
  const int blocks = static_cast<int>(want < cap ? want : cap);
  return launch_pdl(kern, dim3(blocks), dim3(kSmoothThreads), 0, st,
                    static_cast<const uint4*>(a.x), topk_idx,
                    reinterpret_cast<const float4*>(smooth), a.assist, send,
                    static_cast<uint4*>(a.expand_x), a.scales, a.K, a.H, a.A, E);
}

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t st) {
  if (a.bs == 0) return cudaSuccess;
  if (a.quant_mode == 0) {
    const int V = a.H / kVecElems;
    const long long n = static_cast<long long>(a.bs) * V;
    const int per_block = kCopyThreads * kCopyItems;
    const int blocks = static_cast<int>((n + per_block - 1) / per_block);
    const auto kernel = a.K <= 2   ? permute_copy_kernel<2>
                        : a.K <= 4 ? permute_copy_kernel<4>
                        : a.K <= 8 ? permute_copy_kernel<8>
                                   : permute_copy_kernel<16>;
    return launch_pdl(kernel, dim3(blocks), dim3(kCopyThreads), 0, st,
                      static_cast<const uint4*>(a.x), a.assist, static_cast<uint4*>(a.expand_x),
                      a.bs, a.K, V, a.A);
  }
  int threads, cpt;
  quant_shape(a.H, &threads, &cpt);
  const uint4* x = static_cast<const uint4*>(a.x);
  uint4* out = static_cast<uint4*>(a.expand_x);
  const bool bf = a.dtype == MOE_BF16;
  // a persistent grid of as many CTAs as are resident at once (each walks its
  // tokens with the next row in flight), so no partial second wave
  auto launch = [&](auto kernel) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0) != cudaSuccess ||
        per_sm < 1)
      per_sm = 1;
    const int cap = sm_count() * per_sm;
    const int blocks = a.bs < cap ? a.bs : cap;
    return launch_pdl(kernel, dim3(blocks), dim3(threads), 0, st, x, a.assist, out, a.scales,
                      a.bs, a.K, a.H, a.A);
  };
  if (cpt <= 1) return launch(bf ? permute_quant_kernel<Bf16, 1> : permute_quant_kernel<Fp16, 1>);
  if (cpt <= 2) return launch(bf ? permute_quant_kernel<Bf16, 2> : permute_quant_kernel<Fp16, 2>);
  return launch(bf ? permute_quant_kernel<Bf16, 4> : permute_quant_kernel<Fp16, 4>);
}

}  // namespace moe
