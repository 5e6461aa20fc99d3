// Log-sum-exp merge of two partial attention results (HBM-bound).
//
// The vLLM MLA prefill backend computes new-token attention
// (run_prefill_new_tokens, causal) and context-chunk attention
// (run_prefill_context_chunk, unmasked, LSE returned) separately; their
// combination over the union of the key sets is the log-sum-exp identity the
// split-KV combine kernels of the FA4 interface page and the Mojo mla module
// (mla_splitk_reduce) apply:
//   lse = m + ln(e^(lse_a - m) + e^(lse_b - m)),  m = max(lse_a, lse_b)
//   out = e^(lse_a - lse) o_a + e^(lse_b - lse) o_b
//
// Layout: o_* [T, H, D] bf16 rows of D elements, lse_* [H, T] fp32.  `out`
// may be o_a or o_b (each element is read, then written, by one thread);
// lse_out must not overlap lse_a/lse_b (other threads still read them).  One
// thread handles one 16-byte vector (8 elements) of one (token, head) row;
// a grid-stride loop covers all T*H*D/8 vectors with two vectors in flight
// per thread.
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace mla {
namespace merge {

constexpr int kThreads = 256;

__device__ __forceinline__ void weights(float la, float lb, float& wa, float& wb, float& lse) {
  const float m = fmaxf(la, lb);
  if (m == -INFINITY) {  // both sides saw no key (NaN inputs fall through)
    wa = 0.f;
    wb = 0.f;
    lse = -INFINITY;
    return;
  }
  const float ea = exp2f((la - m) * 1.4426950408889634f);
  const float eb = exp2f((lb - m) * 1.4426950408889634f);
  const float s = ea + eb;
  const float inv = 1.0f / s;
  wa = ea * inv;
  wb = eb * inv;
  lse = m + logf(s);
}

__device__ __forceinline__ uint4 combine(uint4 a, uint4 b, float wa, float wb) {
  const uint32_t av[4] = {a.x, a.y, a.z, a.w};
  const uint32_t bv[4] = {b.x, b.y, b.z, b.w};
  uint32_t r[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[i]));
    const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bv[i]));
    r[i] = pack_bf16x2(fmaf(wa, fa.x, wb * fb.x), fmaf(wa, fa.y, wb * fb.y));
  }
  return make_uint4(r[0], r[1], r[2], r[3]);
}

__global__ void __launch_bounds__(kThreads)
    merge_kernel(const uint4* oa, const float* __restrict__ la, const uint4* ob,
                 const float* __restrict__ lb, uint4* out,
                 float* lse_out, long long num_rows, int num_heads, int num_tokens,
                 int vec_per_row) {
  const long long total = num_rows * vec_per_row;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  // Two independent vectors per iteration to keep more loads in flight.
  for (; i + stride < total; i += 2 * stride) {
    const long long j = i + stride;
    const long long ri = i / vec_per_row, rj = j / vec_per_row;
    const int ti = static_cast<int>(ri / num_heads), hi = static_cast<int>(ri % num_heads);
    const int tj = static_cast<int>(rj / num_heads), hj = static_cast<int>(rj % num_heads);
    const size_t li = static_cast<size_t>(hi) * num_tokens + ti;
    const size_t lj = static_cast<size_t>(hj) * num_tokens + tj;
    const uint4 a0 = oa[i], b0 = ob[i], a1 = oa[j], b1 = ob[j];
    const float la0 = la[li], lb0 = lb[li], la1 = la[lj], lb1 = lb[lj];
    float wa0, wb0, l0, wa1, wb1, l1;
    weights(la0, lb0, wa0, wb0, l0);
    weights(la1, lb1, wa1, wb1, l1);
    out[i] = combine(a0, b0, wa0, wb0);
    out[j] = combine(a1, b1, wa1, wb1);
    if (lse_out != nullptr) {
      if (i % vec_per_row == 0) lse_out[li] = l0;
      if (j % vec_per_row == 0) lse_out[lj] = l1;
    }
  }
  for (; i < total; i += stride) {
    const long long ri = i / vec_per_row;
    const int ti = static_cast<int>(ri / num_heads), hi = static_cast<int>(ri % num_heads);
    const size_t li = static_cast<size_t>(hi) * num_tokens + ti;
    float wa, wb, l;
    weights(la[li], lb[li], wa, wb, l);
    out[i] = combine(oa[i], ob[i], wa, wb);
    if (lse_out != nullptr && i % vec_per_row == 0) lse_out[li] = l;
  }
}

}  // namespace merge
}  // namespace mla

namespace mla {
namespace merge {

// Split-KV combine: the N-way form of the merge above (the combine step of
// the split-KV path the FA4 interface page describes, and of the Mojo mla
// module's mla_splitk_reduce).  For each (token, head) row with partial
// results (O_s, lse_s), s < nsplit, over disjoint key ranges:
//   lse = m + ln sum_s e^(lse_s - m),  m = max_s lse_s
//   out = sum_s e^(lse_s - lse) O_s
// A split without keys has lse_s = -inf (weight 0); a row without any key
// gets out = 0, lse = -inf.  Partials: o_part fp32 [nsplit][T][H][128],
// lse_part [nsplit][H][T]; out bf16 [T][H][128], lse [H][T] (may be null).
// One warp per row, four dims per lane.
constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads)
    combine_splits_kernel(const float4* __restrict__ o_part, const float* __restrict__ lse_part,
                          int nsplit, int num_tokens, int num_heads, uint2* out, float* lse) {
  const long long rows = static_cast<long long>(num_tokens) * num_heads;
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       row < rows; row += warps) {
    const int t = static_cast<int>(row / num_heads), h = static_cast<int>(row % num_heads);
    const size_t li = static_cast<size_t>(h) * num_tokens + t;
    const size_t split_lse = static_cast<size_t>(num_heads) * num_tokens;
    float m = -INFINITY;
    for (int s = 0; s < nsplit; ++s) m = fmaxf(m, lse_part[s * split_lse + li]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float z = 0.f;
    if (m != -INFINITY) {
      for (int s = 0; s < nsplit; ++s) {
        const float w = exp2f((lse_part[s * split_lse + li] - m) * 1.4426950408889634f);
        const float4 o = o_part[(static_cast<size_t>(s) * rows + row) * 32 + lane];
        acc.x = fmaf(w, o.x, acc.x);
        acc.y = fmaf(w, o.y, acc.y);
        acc.z = fmaf(w, o.z, acc.z);
        acc.w = fmaf(w, o.w, acc.w);
        z += w;
      }
    }
    const float inv = z > 0.f ? 1.0f / z : 0.f;
    out[row * 32 + lane] = make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv),
                                      pack_bf16x2(acc.z * inv, acc.w * inv));
    if (lse != nullptr && lane == 0) lse[li] = z > 0.f ? m + logf(z) : -INFINITY;
  }
}

}  // namespace merge
}  // namespace mla
