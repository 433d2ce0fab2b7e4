// Dispatch permute: expand_x[slot(t, k)] = x[t] for every pair with a slot,
// optionally quantised to int8 per token ([combine] Parameters:
// comm_quant_mode 2; Example: quant_mode = 2).
//
// Plain copy: one thread per 16-byte vector of x (coalesced along the row),
// read once and stored to each of the token's K slots; one-shot blocks.
//
// int8: one CTA per token (grid-stride); each thread keeps 16-element chunks
// of the row in registers, the CTA reduces max|x|, and every chunk becomes one
// 16-byte int8 store per slot.
#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int kCopyThreads = 256;
constexpr int kCopyItems = 2;  // vectors per thread, a block apart

// One thread per 16-byte vector of x (coalesced along the row) in one-shot
// blocks: the vector is read once and stored to each of the token's K slots.
__global__ void __launch_bounds__(kCopyThreads) permute_copy_kernel(
    const uint4* __restrict__ x, const int32_t* __restrict__ assist, uint4* __restrict__ out,
    int bs, int K, int V, int A) {
  pdl_trigger();
  pdl_wait();
  const int n = bs * V;
  const int32_t* slots_all = assist + static_cast<size_t>(A);
#pragma unroll
  for (int i = 0; i < kCopyItems; ++i) {
    const int item = (blockIdx.x * kCopyItems + i) * kCopyThreads + threadIdx.x;
    if (item >= n) return;
    const int t = item / V;
    const int v = item - t * V;
    const uint4 val = ld_nc_v4(x + item);
    const int32_t* slots = slots_all + static_cast<size_t>(t) * K;
    for (int k = 0; k < K; ++k) {
      const int s = __ldg(slots + k);
      if (s >= 0) st_v4(out + static_cast<size_t>(s) * V + v, val);
    }
  }
}

// CPT 16-element chunks per thread (1, 2 or 4), chosen by the launcher so a
// row fits the CTA with as few registers as possible.
template <typename T16, int CPT>
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
    const int32_t* slots = assist + static_cast<size_t>(A) + static_cast<size_t>(t) * K;
    const int my_slot = lane < K ? __ldg(slots + lane) : -1;  // every warp holds the K slots
    float f[CPT][16];
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
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
    const float inv_scale = 1.0f / scale;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int c = threadIdx.x + j * blockDim.x;
      const bool mine = c < C;  // every lane still takes part in the shuffles below
      uint32_t packed[4];
#pragma unroll
      for (int w4 = 0; w4 < 4; ++w4) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          int q = 0;
          if (mine && amax != 0.0f) {
            float r = quant_code(f[j][w4 * 4 + b], scale, inv_scale);
            r = fminf(127.0f, fmaxf(-127.0f, r));
            q = __float2int_rn(r);
          }
          word |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * b);
        }
        packed[w4] = word;
      }
      const uint4 val = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      for (int k = 0; k < K; ++k) {
        const int s = __shfl_sync(0xFFFFFFFFu, my_slot, k);
        if (mine && s >= 0) st_v4(out + static_cast<size_t>(s) * C + c, val);
      }
    }
    if (warp == 0 && lane < K && my_slot >= 0) scales[my_slot] = scale;
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

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t st) {
  if (a.bs == 0) return cudaSuccess;
  if (a.quant_mode == 0) {
    const int V = a.H / kVecElems;
    const long long n = static_cast<long long>(a.bs) * V;
    const int per_block = kCopyThreads * kCopyItems;
    const int blocks = static_cast<int>((n + per_block - 1) / per_block);
    return launch_pdl(permute_copy_kernel, dim3(blocks), dim3(kCopyThreads), 0, st,
                      static_cast<const uint4*>(a.x), a.assist, static_cast<uint4*>(a.expand_x),
                      a.bs, a.K, V, a.A);
  }
  int threads, cpt;
  quant_shape(a.H, &threads, &cpt);
  const int cap = sm_count() * (2048 / threads);
  const int blocks = a.bs < cap ? a.bs : cap;
  const uint4* x = static_cast<const uint4*>(a.x);
  uint4* out = static_cast<uint4*>(a.expand_x);
  const bool bf = a.dtype == MOE_BF16;
  if (cpt <= 1)
    return launch_pdl(bf ? permute_quant_kernel<Bf16, 1> : permute_quant_kernel<Fp16, 1>,
                      dim3(blocks), dim3(threads), 0, st, x, a.assist, out, a.scales, a.bs, a.K,
                      a.H, a.A);
  if (cpt <= 2)
    return launch_pdl(bf ? permute_quant_kernel<Bf16, 2> : permute_quant_kernel<Fp16, 2>,
                      dim3(blocks), dim3(threads), 0, st, x, a.assist, out, a.scales, a.bs, a.K,
                      a.H, a.A);
  return launch_pdl(bf ? permute_quant_kernel<Bf16, 4> : permute_quant_kernel<Fp16, 4>,
                    dim3(blocks), dim3(threads), 0, st, x, a.assist, out, a.scales, a.bs, a.K,
                    a.H, a.A);
}

}  // namespace moe
