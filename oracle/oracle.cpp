// Plain, slow CPU oracle for MoE token dispatch and combine on one device.
//
// TEST INFRASTRUCTURE. Only the tests, the package's smoke entry and the
// benchmark's CPU-baseline leg may load this library. The CUDA path never
// calls it, includes it or shares any code, header or table with it.
//
// What it follows (page titles and sections):
//   [combine]  Ascend CANN "low_latency_combine" API page: Function
//              (Description, Formula, special expert use cases), Parameters
//              table, Constraints, Deterministic Computation, Example
//              (single-operator mode call).
//   [ep_moe]   Triton-distributed PR "Modify ep_moe_fused 's backward to run
//              with ep_size < 8": the fused EP MoE layer has a backward, which
//              the combine backward below serves.
//
// Threads: built plain (the pinned build the tests check), every function is
// single-threaded. Built with -fopenmp (the benchmark's all-cores CPU timing
// only), the per-token loops that write disjoint outputs run their tokens on
// all cores; each token's arithmetic, and so every result, is unchanged.
//
// Precision: the pages fix bf16/fp16 storage and fp32 topk_weights; the combine
// accumulation is fp32, every product and every sum rounded on its own (this
// file is compiled with -ffp-contract=off), in k order. grad_w is summed in
// double and rounded to fp32 once, so it serves as the accurate side of the
// relative-error check.
//
// Readings of points the pages leave open (each one is also listed with its
// reason in the design notes):
//   R1 shared_expert_x is added once, unweighted, after the weighted k sum.
//   R2 special-expert outputs (zero/copy/const) are weighted by topk_weights
//      like routed ones.
//   R3 special experts get no slot in the expanded buffer and are not counted.
//   R4 const expert j = id - (E + Z + C) uses row j of alpha_1, alpha_2 and v.
//   R5 ep_send_counts is the exclusive prefix sum with the total appended
//      (E + 1 entries).
//   R6 assist_info is a buffer of A + BS*K int32: entry s < A holds t*K + k of
//      the pair in slot s (or -1 when s >= R), entry A + t*K + k holds the slot
//      of pair (t, k) (or -1 when the pair has no slot).
//   R7 inside an expert's segment, pairs are ordered by token, then k (a stable
//      sort of the (t, k)-ordered pair list by expert id).
//   R8 a masked pair contributes nothing; shared_expert_x is still added.
//   R9 int8 quantisation: scale = max_h |x| / 127 in fp32, q = clamp(rne(x /
//      scale), -127, 127); an all-zero row gets scale 0 and codes 0.
//   R10 an id outside [0, N) or a repeat of an id earlier in its row makes the
//      pair invalid: it is flagged in the status word and takes no part.
//   R11 grad_w of a pair without a slot (masked, invalid or special) is 0.
//   R17 backward of the special experts (same Formula, local terms): for a
//      copy pair grad_w = <g, ori_x[t]>, for a const pair j
//      grad_w = <g, alpha_1[j] ori_x[t] + alpha_2[j] v[j]> (m as in the forward);
//      grad_ori_x[t] = round16(sum over copy/const pairs, k ascending, of
//      c = fl(w g) for copy and fl(c alpha_1[j]) for const, accumulated in
//      fp32); grad_alpha_1[j] = sum_{t,k} fl(w g) ori_x[t], grad_alpha_2[j] =
//      sum_{t,k} fl(w g) v[j], grad_v[j] = sum_{t,k} fl(w g) alpha_2[j]
//      (fp32 results of double sums). Zero experts contribute nothing.
//   R18 dispatch quantisation with smooth scales (E, H) fp32: the row of pair
//      (t, k) routed to expert e is y = fl(x[t] * scales[e]) (fp32 product),
//      then quantised per row as in R9; each slot has its own codes and scale.
//   R15 combine with comm_quant_mode 2: each expanded row that returns to its
//      token is quantised as in R9 (per row, scale = max|y| / 127) and used as
//      the fp32 value q * scale; special experts and shared_expert_x are local
//      and are not quantised.
//   R19 backward of combine with comm_quant_mode 2: the weighted sum uses the
//      round-trip values D(y) = q * scale, so grad_w[t,k] = <grad_out[t],
//      D(y_slot)> exactly; the round trip itself is piecewise constant and is
//      passed straight through (its Jacobian taken as the identity), so
//      grad_expand = round16(w * grad_out) as without quantisation. The same
//      straight-through reading makes the dispatch-side int8 backward the plain
//      dispatch backward.

#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

enum { ST_BAD_ID = 1, ST_DUP_ID = 2 };
enum { DT_BF16 = 0, DT_FP16 = 1 };

// ---- 16-bit float encodings ------------------------------------------------

float bf16_to_f32(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

uint16_t f32_to_bf16(float f) {
  // Round to nearest even on the upper 16 bits; NaN stays a quiet NaN.
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return static_cast<uint16_t>((u >> 16) | 0x0040u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return static_cast<uint16_t>(u >> 16);
}

float f16_to_f32(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int m = h & 0x3FF;
  float v;
  if (e == 0) {
    v = std::ldexp(static_cast<float>(m), -24);
  } else if (e == 31) {
    v = m ? NAN : INFINITY;
  } else {
    v = std::ldexp(static_cast<float>(m + 1024), e - 25);
  }
  return sign ? -v : v;
}

uint16_t f32_to_f16(float f) {
  // IEEE binary16, round to nearest even, with subnormals and overflow to inf.
  uint32_t u;
  std::memcpy(&u, &f, 4);
  uint16_t sign = static_cast<uint16_t>((u >> 16) & 0x8000u);
  u &= 0x7FFFFFFFu;
  if (u >= 0x7F800000u) return sign | (u > 0x7F800000u ? 0x7E00u : 0x7C00u);
  int e = static_cast<int>(u >> 23);
  if (e == 0) return sign;  // fp32 subnormals are far below half's range
  uint32_t m = (u & 0x7FFFFFu) | 0x800000u;  // value = m * 2^(e - 150)
  int he = e - 112;                           // biased half exponent
  if (he >= 31) return sign | 0x7C00u;
  int shift = he >= 1 ? 13 : 13 + (1 - he);
  if (shift >= 25) return sign;  // below half the smallest subnormal
  uint32_t kept = m >> shift;
  uint32_t rem = m & ((1u << shift) - 1u);
  uint32_t half = 1u << (shift - 1);
  if (rem > half || (rem == half && (kept & 1u))) kept++;
  uint32_t r = he >= 1 ? (static_cast<uint32_t>(he - 1) << 10) + kept : kept;
  if (r >= 0x7C00u) r = 0x7C00u;
  return static_cast<uint16_t>(sign | r);
}

float load16(const uint16_t* p, size_t i, int dtype) {
  return dtype == DT_BF16 ? bf16_to_f32(p[i]) : f16_to_f32(p[i]);
}

uint16_t store16(float f, int dtype) {
  return dtype == DT_BF16 ? f32_to_bf16(f) : f32_to_f16(f);
}

// ---- pair classification ([combine] Parameters: topk_idx, x_active_mask) ----

bool pair_active(const uint8_t* mask, int mask_ndim, int t, int k, int K) {
  if (mask == nullptr || mask_ndim == 0) return true;
  if (mask_ndim == 1) return mask[t] != 0;
  return mask[static_cast<size_t>(t) * K + k] != 0;
}

// 0 = valid; otherwise the status bit that makes it invalid (R10).
int pair_problem(const int32_t* row, int k, int n_ids) {
  int32_t id = row[k];
  if (id < 0 || id >= n_ids) return ST_BAD_ID;
  for (int j = 0; j < k; ++j)
    if (row[j] == id) return ST_DUP_ID;
  return 0;
}

}  // namespace

extern "C" {

// Exposed so the tests can pin the encodings against library conversions.
float oracle_decode16(uint16_t b, int dtype) { return load16(&b, 0, dtype); }
uint16_t oracle_encode16(float f, int dtype) { return store16(f, dtype); }
void oracle_decode16_array(const uint16_t* b, float* f, long n, int dtype) {
  for (long i = 0; i < n; ++i) f[i] = load16(b, i, dtype);
}
void oracle_encode16_array(const float* f, uint16_t* b, long n, int dtype) {
  for (long i = 0; i < n; ++i) b[i] = store16(f[i], dtype);
}

// Threads the per-token loops use: 1 in the plain build.
int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// Dispatch layout. [combine] Parameters (assist_info_for_combine,
// ep_send_counts, x_active_mask), Constraints (A); readings R3, R5-R8, R10.
// Returns the status bits found.
int oracle_dispatch_layout(int bs, int K, int num_experts, int n_ids, int a_capacity,
                           const int32_t* topk_idx, const uint8_t* mask, int mask_ndim,
                           int32_t* expert_token_nums, int32_t* ep_send_counts,
                           int32_t* assist_info) {
  int status = 0;
  struct Pair { int32_t e, t, k; };
  std::vector<Pair> pairs;  // routed active pairs, in (t, k) order
  for (int t = 0; t < bs; ++t) {
    const int32_t* row = topk_idx + static_cast<size_t>(t) * K;
    for (int k = 0; k < K; ++k) {
      int p = pair_problem(row, k, n_ids);
      status |= p;
      if (p) continue;
      if (!pair_active(mask, mask_ndim, t, k, K)) continue;
      if (row[k] >= num_experts) continue;  // special experts take no slot (R3)
      pairs.push_back({row[k], t, k});
    }
  }
  std::stable_sort(pairs.begin(), pairs.end(),
                   [](const Pair& a, const Pair& b) { return a.e < b.e; });
  for (int e = 0; e < num_experts; ++e) expert_token_nums[e] = 0;
  for (const Pair& p : pairs) expert_token_nums[p.e]++;
  ep_send_counts[0] = 0;
  for (int e = 0; e < num_experts; ++e)
    ep_send_counts[e + 1] = ep_send_counts[e] + expert_token_nums[e];
  const size_t A = static_cast<size_t>(a_capacity);
  for (size_t s = 0; s < A + static_cast<size_t>(bs) * K; ++s) assist_info[s] = -1;
  for (size_t s = 0; s < pairs.size(); ++s) {
    int32_t tk = pairs[s].t * K + pairs[s].k;
    assist_info[s] = tk;
    assist_info[A + tk] = static_cast<int32_t>(s);
  }
  return status;
}

// Dispatch permute, no quantisation: expand_x[slot(t, k)] = x[t].
// [combine] Function: the dispatch side collects rows that combine returns
// "along the same path"; at one device the alltoallv is this local copy.
void oracle_dispatch_permute(int bs, int K, int h, int a_capacity, const uint16_t* x,
                             const int32_t* assist_info, uint16_t* expand_x) {
  const size_t A = static_cast<size_t>(a_capacity);
#pragma omp parallel for schedule(static)
  for (int t = 0; t < bs; ++t)
    for (int k = 0; k < K; ++k) {
      int32_t s = assist_info[A + static_cast<size_t>(t) * K + k];
      if (s < 0) continue;
      std::memcpy(expand_x + static_cast<size_t>(s) * h, x + static_cast<size_t>(t) * h,
                  sizeof(uint16_t) * h);
    }
}

// Dispatch permute with dynamic int8 quantisation (quant_mode / comm_quant_mode
// 2 in the Example and the Parameters table); reading R9.
void oracle_dispatch_permute_quant(int bs, int K, int h, int a_capacity, int dtype,
                                   const uint16_t* x, const int32_t* assist_info,
                                   int8_t* expand_q, float* dynamic_scales) {
  std::fesetround(FE_TONEAREST);
  const size_t A = static_cast<size_t>(a_capacity);
#pragma omp parallel for schedule(static)
  for (int t = 0; t < bs; ++t) {
    std::vector<int8_t> codes(h);
    const uint16_t* xr = x + static_cast<size_t>(t) * h;
    float amax = 0.0f;
    for (int j = 0; j < h; ++j) amax = std::max(amax, std::fabs(load16(xr, j, dtype)));
    float scale = amax / 127.0f;
    for (int j = 0; j < h; ++j) {
      if (amax == 0.0f) { codes[j] = 0; continue; }
      float r = std::nearbyint(load16(xr, j, dtype) / scale);
      r = std::min(127.0f, std::max(-127.0f, r));
      codes[j] = static_cast<int8_t>(r);
    }
    for (int k = 0; k < K; ++k) {
      int32_t s = assist_info[A + static_cast<size_t>(t) * K + k];
      if (s < 0) continue;
      std::memcpy(expand_q + static_cast<size_t>(s) * h, codes.data(), h);
      dynamic_scales[s] = scale;
    }
  }
}

// Per-row int8 round trip of R9/R15: max |y| of a row, and the fp32 value
// q * scale of one element given it.
static float row_amax(const uint16_t* row, int h, int dtype) {
  float amax = 0.0f;
  for (int i = 0; i < h; ++i) amax = std::max(amax, std::fabs(load16(row, i, dtype)));
  return amax;
}

static float int8_roundtrip(float y, float amax) {
  if (amax == 0.0f) return 0.0f;
  const float scale = amax / 127.0f;
  float q = std::nearbyint(y / scale);
  q = std::min(127.0f, std::max(-127.0f, q));
  return q * scale;
}

// Dispatch permute with int8 quantisation of smooth-scaled rows (reading
// R18; [combine] Example, graph mode: quant_mode 2 with a scales tensor of
// shape (E, H)).
void oracle_dispatch_permute_quant_smooth(int bs, int K, int h, int a_capacity, int dtype,
                                          const uint16_t* x, const int32_t* topk_idx,
                                          const float* smooth_scales,
                                          const int32_t* assist_info, int8_t* expand_q,
                                          float* dynamic_scales) {
  std::fesetround(FE_TONEAREST);
  const size_t A = static_cast<size_t>(a_capacity);
#pragma omp parallel for schedule(static)
  for (int t = 0; t < bs; ++t) {
    std::vector<float> y(h);
    const uint16_t* xr = x + static_cast<size_t>(t) * h;
    for (int k = 0; k < K; ++k) {
      const int32_t s = assist_info[A + static_cast<size_t>(t) * K + k];
      if (s < 0) continue;
      const int32_t e = topk_idx[static_cast<size_t>(t) * K + k];
      const float* se = smooth_scales + static_cast<size_t>(e) * h;
      float amax = 0.0f;
      for (int j = 0; j < h; ++j) {
        y[j] = load16(xr, j, dtype) * se[j];
        amax = std::max(amax, std::fabs(y[j]));
      }
      const float scale = amax / 127.0f;
      for (int j = 0; j < h; ++j) {
        float r = 0.0f;
        if (amax != 0.0f) {
          r = std::nearbyint(y[j] / scale);
          r = std::min(127.0f, std::max(-127.0f, r));
        }
        expand_q[static_cast<size_t>(s) * h + j] = static_cast<int8_t>(r);
      }
      dynamic_scales[s] = scale;
    }
  }
}

// Combine forward. [combine] Function (Formula: weighted sum of the returned
// rows plus shared_expert_x; special expert use cases: zero, copy, const),
// Parameters (topk_weights, x_active_mask, shared_expert_x, ori_x,
// const_expert_alpha_1/2, const_expert_v, comm_quant_mode), Return Value.
// Readings R1, R2, R4, R8, R10, R15. fp32, product and sum rounded
// separately, k ascending.
void oracle_combine_fwd(int bs, int K, int h, int num_experts, int zero_num, int copy_num,
                        int const_num, int a_capacity, int dtype, const uint16_t* expand_x,
                        const int32_t* topk_idx, const float* topk_weights,
                        const int32_t* assist_info, const uint8_t* mask, int mask_ndim,
                        const uint16_t* shared_x, const uint16_t* ori_x,
                        const uint16_t* alpha1, const uint16_t* alpha2,
                        const uint16_t* const_v, int comm_quant_mode, uint16_t* out) {
  std::fesetround(FE_TONEAREST);
  const size_t A = static_cast<size_t>(a_capacity);
  const int n_ids = num_experts + zero_num + copy_num + const_num;
  const int zero_end = num_experts + zero_num;
  const int copy_end = zero_end + copy_num;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < bs; ++t) {
    std::vector<float> amax(K);
    const int32_t* row = topk_idx + static_cast<size_t>(t) * K;
    if (comm_quant_mode == 2)
      for (int k = 0; k < K; ++k) {
        int32_t s = assist_info[A + static_cast<size_t>(t) * K + k];
        amax[k] = s < 0 ? 0.0f : row_amax(expand_x + static_cast<size_t>(s) * h, h, dtype);
      }
    for (int j = 0; j < h; ++j) {
      float acc = 0.0f;
      for (int k = 0; k < K; ++k) {
        if (pair_problem(row, k, n_ids)) continue;
        if (!pair_active(mask, mask_ndim, t, k, K)) continue;
        const int32_t id = row[k];
        float m;
        if (id < num_experts) {
          int32_t s = assist_info[A + static_cast<size_t>(t) * K + k];
          if (s < 0) continue;
          m = load16(expand_x, static_cast<size_t>(s) * h + j, dtype);
          if (comm_quant_mode == 2) m = int8_roundtrip(m, amax[k]);
        } else if (id < zero_end) {
          m = 0.0f;
        } else if (id < copy_end) {
          m = load16(ori_x, static_cast<size_t>(t) * h + j, dtype);
        } else {
          const size_t q = static_cast<size_t>(id - copy_end);
          float p1 = load16(alpha1, q * h + j, dtype) *
                     load16(ori_x, static_cast<size_t>(t) * h + j, dtype);
          float p2 = load16(alpha2, q * h + j, dtype) * load16(const_v, q * h + j, dtype);
          m = p1 + p2;
        }
        float prod = topk_weights[static_cast<size_t>(t) * K + k] * m;
        acc = acc + prod;
      }
      if (shared_x) acc = acc + load16(shared_x, static_cast<size_t>(t) * h + j, dtype);
      out[static_cast<size_t>(t) * h + j] = store16(acc, dtype);
    }
  }
}

// Combine backward for x = sum_k w[t,k] * expand_x[slot(t,k)] (+ shared):
//   grad_expand[slot(t,k)] = round16(w[t,k] * grad_out[t])  (fp32 product)
//   grad_w[t,k] = sum_h grad_out[t,h] * expand_x[slot(t,k),h]  (double sum)
// abs_sum[t,k] = sum_h |grad_out * expand_x| bounds the rounding error of any
// summation order. Reading R11. The gradient of shared_expert_x is grad_out
// itself and needs no computation.
void oracle_combine_bwd(int bs, int K, int h, int a_capacity, int dtype,
                        const uint16_t* grad_out, const uint16_t* expand_x,
                        const float* topk_weights, const int32_t* assist_info,
                        const uint8_t* mask, int mask_ndim, uint16_t* grad_expand,
                        float* grad_w, double* abs_sum) {
  const size_t A = static_cast<size_t>(a_capacity);
#pragma omp parallel for schedule(static)
  for (int t = 0; t < bs; ++t) {
    const uint16_t* g = grad_out + static_cast<size_t>(t) * h;
    for (int k = 0; k < K; ++k) {
      const size_t tk = static_cast<size_t>(t) * K + k;
      int32_t s = assist_info[A + tk];
      if (s < 0 || !pair_active(mask, mask_ndim, t, k, K)) {
        grad_w[tk] = 0.0f;
        if (abs_sum) abs_sum[tk] = 0.0;
        continue;
      }
      const float w = topk_weights[tk];
      const uint16_t* xr = expand_x + static_cast<size_t>(s) * h;
      uint16_t* ge = grad_expand + static_cast<size_t>(s) * h;
      double dot = 0.0, mag = 0.0;
      for (int j = 0; j < h; ++j) {
        float gj = load16(g, j, dtype);
        ge[j] = store16(w * gj, dtype);
        double term = static_cast<double>(gj) * static_cast<double>(load16(xr, j, dtype));
        dot += term;
        mag += std::fabs(term);
      }
      grad_w[tk] = static_cast<float>(dot);
      if (abs_sum) abs_sum[tk] = mag;
    }
  }
}

// Combine backward with comm_quant_mode 2 (reading R19; [combine] Parameters,
// comm_quant_mode): as oracle_combine_bwd, but the dot product takes each
// element of the returned row through the per-row int8 round trip (R15) the
// forward applied; grad_expand passes the round trip straight through.
void oracle_combine_bwd_comm_quant(int bs, int K, int h, int a_capacity, int dtype,
                                   const uint16_t* grad_out, const uint16_t* expand_x,
                                   const float* topk_weights, const int32_t* assist_info,
                                   const uint8_t* mask, int mask_ndim, uint16_t* grad_expand,
                                   float* grad_w, double* abs_sum) {
  std::fesetround(FE_TONEAREST);
  const size_t A = static_cast<size_t>(a_capacity);
#pragma omp parallel for schedule(static)
  for (int t = 0; t < bs; ++t) {
    const uint16_t* g = grad_out + static_cast<size_t>(t) * h;
    for (int k = 0; k < K; ++k) {
      const size_t tk = static_cast<size_t>(t) * K + k;
      const int32_t s = assist_info[A + tk];
      if (s < 0 || !pair_active(mask, mask_ndim, t, k, K)) {
        grad_w[tk] = 0.0f;
        if (abs_sum) abs_sum[tk] = 0.0;
        continue;
      }
      const float w = topk_weights[tk];
      const uint16_t* yr = expand_x + static_cast<size_t>(s) * h;
      uint16_t* ge = grad_expand + static_cast<size_t>(s) * h;
      const float amax = row_amax(yr, h, dtype);
      double dot = 0.0, mag = 0.0;
      for (int j = 0; j < h; ++j) {
        const float gj = load16(g, j, dtype);
        ge[j] = store16(w * gj, dtype);
        const float d = int8_roundtrip(load16(yr, j, dtype), amax);
        const double term = static_cast<double>(gj) * static_cast<double>(d);
        dot += term;
        mag += std::fabs(term);
      }
      grad_w[tk] = static_cast<float>(dot);
      if (abs_sum) abs_sum[tk] = mag;
    }
  }
}

// Backward of the special experts (reading R17). [combine] Function
// (special expert use cases: copy Moe(ori_x) = ori_x, const Moe(ori_x) =
// alpha_1 ori_x + alpha_2 v) differentiated through the weighted sum of the
// Formula. grad_w gets entries only for copy and const pairs (others are left
// as they are); abs_sum bounds the rounding error of grad_w as in the routed
// backward. grad_ori_x is 16-bit; the alpha/v gradients are fp32 (Q, H) with
// their abs sums for the tolerance.
void oracle_combine_bwd_special(int bs, int K, int h, int num_experts, int zero_num, int copy_num,
                                int const_num, int dtype, const uint16_t* grad_out,
                                const int32_t* topk_idx, const float* topk_weights,
                                const uint8_t* mask, int mask_ndim, const uint16_t* ori_x,
                                const uint16_t* alpha1, const uint16_t* alpha2,
                                const uint16_t* const_v, float* grad_w, double* abs_sum,
                                uint16_t* grad_ori_x, float* grad_alpha1, float* grad_alpha2,
                                float* grad_v, double* abs_alpha1, double* abs_alpha2,
                                double* abs_v) {
  const int n_ids = num_experts + zero_num + copy_num + const_num;
  const int zero_end = num_experts + zero_num, copy_end = zero_end + copy_num;
  const size_t qh = static_cast<size_t>(const_num) * h;
  std::vector<double> ga1(qh, 0.0), ga2(qh, 0.0), gv(qh, 0.0), aa1(qh, 0.0), aa2(qh, 0.0),
      av(qh, 0.0);
  for (int t = 0; t < bs; ++t) {
    const int32_t* row = topk_idx + static_cast<size_t>(t) * K;
    const uint16_t* g = grad_out + static_cast<size_t>(t) * h;
    const uint16_t* ox = ori_x ? ori_x + static_cast<size_t>(t) * h : nullptr;
    for (int k = 0; k < K; ++k) {
      const size_t tk = static_cast<size_t>(t) * K + k;
      if (pair_problem(row, k, n_ids) || !pair_active(mask, mask_ndim, t, k, K)) continue;
      const int32_t id = row[k];
      if (id < zero_end) continue;  // routed (handled elsewhere) or zero expert
      const float w = topk_weights[tk];
      double dot = 0.0, mag = 0.0;
      const size_t q = static_cast<size_t>(id - copy_end);
      for (int j = 0; j < h; ++j) {
        const float gj = load16(g, j, dtype), xj = load16(ox, j, dtype);
        float m;
        if (id < copy_end) {
          m = xj;
        } else {
          const float p1 = load16(alpha1, q * h + j, dtype) * xj;
          const float p2 = load16(alpha2, q * h + j, dtype) * load16(const_v, q * h + j, dtype);
          m = p1 + p2;
          const double c = static_cast<double>(w * gj);
          ga1[q * h + j] += c * xj;
          aa1[q * h + j] += std::fabs(c * xj);
          ga2[q * h + j] += c * load16(const_v, q * h + j, dtype);
          aa2[q * h + j] += std::fabs(c * load16(const_v, q * h + j, dtype));
          gv[q * h + j] += c * load16(alpha2, q * h + j, dtype);
          av[q * h + j] += std::fabs(c * load16(alpha2, q * h + j, dtype));
        }
        const double term = static_cast<double>(gj) * static_cast<double>(m);
        dot += term;
        mag += std::fabs(term);
      }
      grad_w[tk] = static_cast<float>(dot);
      if (abs_sum) abs_sum[tk] = mag;
    }
    for (int j = 0; j < h; ++j) {
      float acc = 0.0f;
      const float gj = load16(g, j, dtype);
      for (int k = 0; k < K; ++k) {
        if (pair_problem(row, k, n_ids) || !pair_active(mask, mask_ndim, t, k, K)) continue;
        const int32_t id = row[k];
        if (id < zero_end) continue;
        const float c = topk_weights[static_cast<size_t>(t) * K + k] * gj;
        if (id < copy_end) {
          acc = acc + c;
        } else {
          const size_t q = static_cast<size_t>(id - copy_end);
          acc = acc + c * load16(alpha1, q * h + j, dtype);
        }
      }
      if (grad_ori_x) grad_ori_x[static_cast<size_t>(t) * h + j] = store16(acc, dtype);
    }
  }
  for (size_t i = 0; i < qh; ++i) {
    grad_alpha1[i] = static_cast<float>(ga1[i]);
    grad_alpha2[i] = static_cast<float>(ga2[i]);
    grad_v[i] = static_cast<float>(gv[i]);
    if (abs_alpha1) abs_alpha1[i] = aa1[i];
    if (abs_alpha2) abs_alpha2[i] = aa2[i];
    if (abs_v) abs_v[i] = av[i];
  }
}

// Dispatch backward: the gradient of the permute's copies returns to each
// token as the unweighted fp32 sum, k ascending, of its slots' gradients.
void oracle_dispatch_bwd(int bs, int K, int h, int a_capacity, int dtype,
                         const uint16_t* grad_in, const int32_t* assist_info,
                         const uint8_t* mask, int mask_ndim, uint16_t* grad_x) {
  const size_t A = static_cast<size_t>(a_capacity);
#pragma omp parallel for schedule(static)
  for (int t = 0; t < bs; ++t)
    for (int j = 0; j < h; ++j) {
      float acc = 0.0f;
      for (int k = 0; k < K; ++k) {
        int32_t s = assist_info[A + static_cast<size_t>(t) * K + k];
        if (s < 0 || !pair_active(mask, mask_ndim, t, k, K)) continue;
        acc = acc + load16(grad_in, static_cast<size_t>(s) * h + j, dtype);
      }
      grad_x[static_cast<size_t>(t) * h + j] = store16(acc, dtype);
    }
}

}  // extern "C"
