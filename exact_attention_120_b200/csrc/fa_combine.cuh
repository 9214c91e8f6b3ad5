// Merge of the split-key partial results of the attention forward pass.
//
// Each key slice s of a query row produced a normalised partial output O_s
// and its logsumexp lse_s = m_s + ln l_s.  The row's result follows from the
// concatenated-softmax rule of "理解 Flash Attention" (section "瓦片注意力计算"):
// with m = max_s lse_s and w_s = exp(lse_s - m),
//     O = sum_s w_s O_s / sum_s w_s,    lse = m + ln sum_s w_s,
// because w_s is proportional to the slice's share e^{m_s} l_s of the row's
// softmax denominator.  Slices that saw no key have lse_s = -inf and weight 0;
// a row with no key at all gets O = 0, lse = -inf.
//
// One warp per query row; lane t owns columns [t * D/32, (t+1) * D/32).  The
// kernel only streams the workspace (splits x (D + 1) floats per row), so it is
// bound by HBM bandwidth.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace fa {

template <int D>
__global__ void __launch_bounds__(256) fa_combine_kernel(const float* __restrict__ part_o,
                                                         const float* __restrict__ part_lse,
                                                         __nv_bfloat16* __restrict__ o,
                                                         float* __restrict__ lse, long long rows,
                                                         int splits) {
  constexpr int kCols = D / 32;  // columns per lane: 4 (d=128) or 2 (d=64)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the partials of the split launch
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float m = -INFINITY;
  for (int s = lane; s < splits; s += 32) m = fmaxf(m, part_lse[(long long)s * rows + row]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float acc[kCols];
#pragma unroll
  for (int i = 0; i < kCols; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < splits; ++s) {
      const float ls = part_lse[(long long)s * rows + row];
      if (ls == -INFINITY) continue;
      const float w = __expf(ls - m);
      wsum += w;
      const float* src = part_o + ((long long)s * rows + row) * D + lane * kCols;
      if constexpr (kCols == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        acc[0] += w * v.x;
        acc[1] += w * v.y;
        acc[2] += w * v.z;
        acc[3] += w * v.w;
      } else {
        const float2 v = *reinterpret_cast<const float2*>(src);
        acc[0] += w * v.x;
        acc[1] += w * v.y;
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* dst = o + row * D + lane * kCols;
#pragma unroll
  for (int i = 0; i < kCols; i += 2)
    *reinterpret_cast<__nv_bfloat162*>(dst + i) = __floats2bfloat162_rn(acc[i] * inv, acc[i + 1] * inv);
  if (lane == 0) lse[row] = wsum > 0.f ? m + __logf(wsum) : -INFINITY;
}

}  // namespace fa
