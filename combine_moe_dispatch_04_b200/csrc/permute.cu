// Dispatch permute: expand_x[slot(t, k)] = x[t] for every pair with a slot,
// optionally quantised to int8 per token ([combine] Parameters:
// comm_quant_mode 2; Example: quant_mode = 2).
//
// Plain copy: one thread per 16-byte vector of x (coalesced along the row),
// read once and stored to each of the token's K slots. The slot list of a
// token is shared by the threads of its row and comes from L1.
//
// int8: one CTA per token (grid-stride); each thread keeps 16-element chunks
// of the row in registers, the CTA reduces max|x|, and every chunk becomes one
// 16-byte int8 store per slot.
#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int kCopyThreads = 256;
constexpr int kCopyWarps = kCopyThreads / 32;
constexpr int kCopyU = 2;  // vectors per lane per item

// One warp per (token, chunk of 32 * kCopyU vectors) item over a persistent
// grid: the chunk of x[t] is read once into registers and stored to each of
// the token's slots. Lane k < K holds slot k and broadcasts it by shuffle.
__global__ void __launch_bounds__(kCopyThreads) permute_copy_kernel(
    const uint4* __restrict__ x, const int32_t* __restrict__ assist, uint4* __restrict__ out,
    int K, int V, int A, int chunks, int n_items) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int stride = gridDim.x * kCopyWarps;
  for (int item = blockIdx.x * kCopyWarps + (threadIdx.x >> 5); item < n_items; item += stride) {
    const int t = item / chunks;
    const int v0 = (item - t * chunks) * 32 * kCopyU + lane;
    const int my_slot =
        lane < K ? __ldg(assist + static_cast<size_t>(A) + static_cast<size_t>(t) * K + lane) : -1;
    uint4 val[kCopyU];
#pragma unroll
    for (int u = 0; u < kCopyU; ++u) {
      const int v = v0 + u * 32;
      if (v < V) val[u] = ld_nc_v4(x + static_cast<size_t>(t) * V + v);
    }
    for (int k = 0; k < K; ++k) {
      const int s = __shfl_sync(0xFFFFFFFFu, my_slot, k);
      if (s < 0) continue;
#pragma unroll
      for (int u = 0; u < kCopyU; ++u) {
        const int v = v0 + u * 32;
        if (v < V) st_v4(out + static_cast<size_t>(s) * V + v, val[u]);
      }
    }
  }
}

constexpr int kQuantChunksPerThread = 4;  // 16-element chunks per thread

template <typename T16>
__global__ void __launch_bounds__(256) permute_quant_kernel(
    const uint4* __restrict__ x, const int32_t* __restrict__ assist, uint4* __restrict__ out,
    float* __restrict__ scales, int bs, int K, int H, int A) {
  __shared__ float warp_max[8];
  pdl_trigger();
  pdl_wait();
  const int C = H / 16;  // chunks per row
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  for (int t = blockIdx.x; t < bs; t += gridDim.x) {
    const uint4* xr = x + static_cast<size_t>(t) * (H / 8);
    float f[kQuantChunksPerThread][16];
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < kQuantChunksPerThread; ++j) {
      const int c = threadIdx.x + j * blockDim.x;
      if (c < C) {
        float lo[8], hi[8];
        widen8<T16>(ld_nc_v4(xr + 2 * c), lo);
        widen8<T16>(ld_nc_v4(xr + 2 * c + 1), hi);
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
    if (lane == 0) warp_max[warp] = amax;
    __syncthreads();
    amax = warp_max[0];
    for (int w = 1; w < nwarps; ++w) amax = fmaxf(amax, warp_max[w]);
    __syncthreads();  // warp_max is reused by the next token
    const float scale = __fdiv_rn(amax, 127.0f);
    const int32_t* slots = assist + static_cast<size_t>(A) + static_cast<size_t>(t) * K;
#pragma unroll
    for (int j = 0; j < kQuantChunksPerThread; ++j) {
      const int c = threadIdx.x + j * blockDim.x;
      if (c >= C) continue;
      uint32_t packed[4];
#pragma unroll
      for (int w4 = 0; w4 < 4; ++w4) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          int q = 0;
          if (amax != 0.0f) {
            float r = rintf(__fdiv_rn(f[j][w4 * 4 + b], scale));
            r = fminf(127.0f, fmaxf(-127.0f, r));
            q = __float2int_rn(r);
          }
          word |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * b);
        }
        packed[w4] = word;
      }
      const uint4 val = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      for (int k = 0; k < K; ++k) {
        const int s = __ldg(slots + k);
        if (s >= 0) st_v4(out + static_cast<size_t>(s) * C + c, val);
      }
    }
    if (threadIdx.x < K) {
      const int s = __ldg(slots + threadIdx.x);
      if (s >= 0) scales[s] = scale;
    }
  }
}

}  // namespace

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t st) {
  if (a.bs == 0) return cudaSuccess;
  if (a.quant_mode == 0) {
    const int V = a.H / kVecElems;
    const int chunks = (V + 32 * kCopyU - 1) / (32 * kCopyU);
    const long long items = static_cast<long long>(a.bs) * chunks;
    const long long want = (items + kCopyWarps - 1) / kCopyWarps;
    static int per_sm = 0;
    if (per_sm == 0) {
      int n = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, permute_copy_kernel, kCopyThreads, 0) !=
              cudaSuccess || n < 1)
        n = 1;
      per_sm = n;
    }
    const long long cap = static_cast<long long>(sm_count()) * per_sm;
    const int blocks = static_cast<int>(want < cap ? want : cap);
    return launch_pdl(permute_copy_kernel, dim3(blocks), dim3(kCopyThreads), 0, st,
                      static_cast<const uint4*>(a.x), a.assist, static_cast<uint4*>(a.expand_x),
                      a.K, V, a.A, chunks, static_cast<int>(items));
  }
  // One chunk per thread up to 256 threads, then up to 4 chunks per thread
  // (H <= 16384, checked by the caller).
  const int C = a.H / 16;
  int threads = (C + 31) / 32 * 32;
  threads = threads > 256 ? 256 : threads;
  const int cap = sm_count() * 16;
  const int blocks = a.bs < cap ? a.bs : cap;
  auto kernel = a.dtype == MOE_BF16 ? permute_quant_kernel<Bf16> : permute_quant_kernel<Fp16>;
  return launch_pdl(kernel, dim3(blocks), dim3(threads), 0, st, static_cast<const uint4*>(a.x),
                    a.assist, static_cast<uint4*>(a.expand_x), a.scales, a.bs, a.K, a.H, a.A);
}

}  // namespace moe
