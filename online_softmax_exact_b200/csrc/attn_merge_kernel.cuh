// attn_merge_kernel.cuh - merge of partial attention results (O_i, LSE_i) computed
// over disjoint key sets.
//
// Per row, with M = max_i LSE_i and w_i = exp(LSE_i - M):
//   O = sum_i w_i O_i / sum_i w_i,  LSE = M + ln(sum_i w_i).
// This is the rescale-to-a-common-maximum step of the online softmax ("FlashAttention
// by hand", paragraphs on the running statistics and rescaling) applied to whole
// partial results; ATTENTION2D (sections 2 and 3) combines fragment statistics this
// way and relies on the combination being commutative and associative.
//
// The kernel is a pure HBM stream: each row's d fp32 values are read once per part
// with 128-bit loads (D/4 threads per row, consecutive threads on consecutive 16-byte
// chunks) and written once; LSEs are read by every thread of the row (one broadcast
// transaction per warp). Grid-stride over rows; all part loads of a row are issued
// before they are consumed.
#pragma once

#include <cstdint>

namespace osx {

constexpr int kMaxMergeParts = 64;

struct MergeParams {
  const float* o[kMaxMergeParts];
  const float* lse[kMaxMergeParts];
  float* out_o;
  float* out_lse;
  long long rows;
  int n;
};

__device__ __forceinline__ float ex2_merge(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float4 ld_stream4(const float* p) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

template <int D>
__global__ void __launch_bounds__(256)
attn_merge_kernel(const __grid_constant__ MergeParams p) {
  constexpr int TPR = D / 4;               // threads per row
  constexpr int RPB = 256 / TPR;           // rows per block per iteration
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr float kLn2 = 0.69314718055994530942f;
  const int sub = threadIdx.x / TPR;
  const int c4 = threadIdx.x % TPR;
  const long long stride = (long long)gridDim.x * RPB;

  for (long long row = (long long)blockIdx.x * RPB + sub; row < p.rows; row += stride) {
    float M = -INFINITY;
    for (int i = 0; i < p.n; ++i) M = fmaxf(M, __ldg(p.lse[i] + row));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
    if (M != -INFINITY) {
      int i = 0;
      for (; i + 4 <= p.n; i += 4) {
        float4 v[4];
        float w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = ld_stream4(p.o[i + u] + row * D + c4 * 4);
#pragma unroll
        for (int u = 0; u < 4; ++u) w[u] = ex2_merge((__ldg(p.lse[i + u] + row) - M) * kLog2e);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          acc.x = fmaf(w[u], v[u].x, acc.x);
          acc.y = fmaf(w[u], v[u].y, acc.y);
          acc.z = fmaf(w[u], v[u].z, acc.z);
          acc.w = fmaf(w[u], v[u].w, acc.w);
          wsum += w[u];
        }
      }
      for (; i < p.n; ++i) {
        const float4 v = ld_stream4(p.o[i] + row * D + c4 * 4);
        const float w = ex2_merge((__ldg(p.lse[i] + row) - M) * kLog2e);
        acc.x = fmaf(w, v.x, acc.x);
        acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z);
        acc.w = fmaf(w, v.w, acc.w);
        wsum += w;
      }
      const float inv = 1.f / wsum;
      acc.x *= inv;
      acc.y *= inv;
      acc.z *= inv;
      acc.w *= inv;
    }
    __stcs(reinterpret_cast<float4*>(p.out_o + row * D + c4 * 4), acc);
    if (c4 == 0) {
      float lse = -INFINITY;
      if (M != -INFINITY) {
        float lg;
        asm("lg2.approx.f32 %0, %1;" : "=f"(lg) : "f"(wsum));
        lse = M + lg * kLn2;
      }
      p.out_lse[row] = lse;
    }
  }
}

}  // namespace osx
