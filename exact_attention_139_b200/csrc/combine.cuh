// combine.cuh -- log-sum-exp merge of split-KV partials.
//
// Chunks cover disjoint key ranges, so with per-chunk results (O_s normalised by its own sum,
// lse_s = ln of its sum) the whole-row result is LSE = ln sum_s exp(lse_s) and
// O = sum_s exp(lse_s - LSE) * O_s. A chunk with lse_s = -inf has no visible key and no weight.
// One CTA per query row; threads stride over the dv columns, four at a time. With the balanced
// decode schedule (bal_w > 0) the number of partials differs per unit (R rows each): the CTAs
// that cover keys u * Lk .. (u + 1) * Lk - 1, each bal_w keys wide, one partial apiece.
#pragma once

#include "sm100.cuh"

namespace attn {

constexpr int kCombineThreads = 128;

template <typename E>
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                   uint16_t* __restrict__ o, float* __restrict__ lse, long long rows, int dv,
                   int num_splits, int bal_w, int Lk, int R) {
  // launched as a programmatic dependent of the decode kernel: wait until that grid has finished
  // and its partials are visible (returns at once for an ordinary launch)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const long long row = blockIdx.x;
  if (bal_w > 0) {
    const long long u = row / R;
    num_splits = (int)(((u + 1) * Lk - 1) / bal_w - (u * Lk) / bal_w + 1);
  }
  float m = -INFINITY;
  for (int s = 0; s < num_splits; ++s) m = fmaxf(m, lse_part[(long long)s * rows + row]);
  float L = -INFINITY;
  if (m != -INFINITY) {
    float sum = 0.f;
    for (int s = 0; s < num_splits; ++s) {
      const float ls = lse_part[(long long)s * rows + row];
      if (ls != -INFINITY) sum += expf(ls - m);
    }
    L = m + logf(sum);
  }
  for (int c = 4 * threadIdx.x; c < dv; c += 4 * kCombineThreads) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (L != -INFINITY) {
      for (int s = 0; s < num_splits; ++s) {
        const float ls = lse_part[(long long)s * rows + row];
        if (ls == -INFINITY) continue;
        const float w = expf(ls - L);
        const float4 x = *reinterpret_cast<const float4*>(o_part + ((long long)s * rows + row) * dv + c);
        acc.x = fmaf(w, x.x, acc.x);
        acc.y = fmaf(w, x.y, acc.y);
        acc.z = fmaf(w, x.z, acc.z);
        acc.w = fmaf(w, x.w, acc.w);
      }
    }
    uint2 packed = make_uint2(E::pack2(acc.x, acc.y), E::pack2(acc.z, acc.w));
    *reinterpret_cast<uint2*>(o + row * dv + c) = packed;
  }
  if (threadIdx.x == 0 && lse != nullptr) lse[row] = L;
}

}  // namespace attn
