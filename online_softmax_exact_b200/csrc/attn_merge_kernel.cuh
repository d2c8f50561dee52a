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
// The kernel is a pure HBM stream: every part's row is read once with 256-bit loads
// (D/8 threads per row, consecutive threads on consecutive 32-byte chunks) and the
// result written once. Parts are taken in groups of G: all loads of a group (O chunks
// and LSEs) for R rows are issued before any is used, so each thread has G*R = 8
// 32-byte loads in flight; each group is folded into a running (max, weight sum,
// weighted sum) - the same online rescale - so any number of parts streams in one
// pass. G is 2, 4 or 8 by the number of parts (R = 8 / G).
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

struct F8 {
  float v[8];
};

__device__ __forceinline__ F8 ld_stream8(const float* p) {
  F8 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=f"(r.v[0]), "=f"(r.v[1]), "=f"(r.v[2]), "=f"(r.v[3]), "=f"(r.v[4]),
                 "=f"(r.v[5]), "=f"(r.v[6]), "=f"(r.v[7])
               : "l"(p));
  return r;
}

__device__ __forceinline__ void st_stream8(float* p, const float (&a)[8]) {
  asm volatile("st.global.cs.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "f"(a[0]),
               "f"(a[1]), "f"(a[2]), "f"(a[3]), "f"(a[4]), "f"(a[5]), "f"(a[6]), "f"(a[7])
               : "memory");
}

template <int D, int G>
__global__ void __launch_bounds__(256)
attn_merge_kernel(const __grid_constant__ MergeParams p) {
  constexpr int TPR = D / 8;  // threads per row, 8 floats each
  constexpr int RPB = 256 / TPR;
  constexpr int R = 8 / G;    // rows in flight per thread
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr float kLn2 = 0.69314718055994530942f;
  const int sub = threadIdx.x / TPR;
  const int c8 = threadIdx.x % TPR;
  const long long step = (long long)gridDim.x * RPB;

  for (long long row0 = (long long)blockIdx.x * RPB + sub; row0 < p.rows; row0 += R * step) {
    float M[R], wsum[R], acc[R][8];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      M[r] = -INFINITY;
      wsum[r] = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[r][e] = 0.f;
    }
    for (int g0 = 0; g0 < p.n; g0 += G) {
      const int gn = (p.n - g0) < G ? (p.n - g0) : G;
      F8 v[R][G];
      float ls[R][G];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const long long row = row0 + r * step;
#pragma unroll
        for (int i = 0; i < G; ++i) {
          if (i < gn && row < p.rows) {
            v[r][i] = ld_stream8(p.o[g0 + i] + row * D + c8 * 8);
            ls[r][i] = __ldg(p.lse[g0 + i] + row);
          } else {
            ls[r][i] = -INFINITY;
#pragma unroll
            for (int e = 0; e < 8; ++e) v[r][i].v[e] = 0.f;
          }
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float Mg = M[r];
#pragma unroll
        for (int i = 0; i < G; ++i) Mg = fmaxf(Mg, ls[r][i]);
        if (Mg == -INFINITY) continue;  // no keys in any part so far
        // bring the running sums to the new maximum (factor 0 when M was -inf)
        const float a = (Mg == M[r]) ? 1.f : ex2_merge((M[r] - Mg) * kLog2e);
        wsum[r] *= a;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[r][e] *= a;
#pragma unroll
        for (int i = 0; i < G; ++i) {
          const float w = ex2_merge((ls[r][i] - Mg) * kLog2e);  // 0 for empty parts
          wsum[r] += w;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[r][e] = fmaf(w, v[r][i].v[e], acc[r][e]);
        }
        M[r] = Mg;
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const long long row = row0 + r * step;
      if (row >= p.rows) continue;
      const bool empty = (M[r] == -INFINITY);
      const float inv = empty ? 0.f : 1.f / wsum[r];
      float out[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) out[e] = acc[r][e] * inv;
      st_stream8(p.out_o + row * D + c8 * 8, out);
      if (c8 == 0) {
        float lse = -INFINITY;
        if (!empty) {
          float lg;
          asm("lg2.approx.f32 %0, %1;" : "=f"(lg) : "f"(wsum[r]));
          lse = M[r] + lg * kLn2;
        }
        p.out_lse[row] = lse;
      }
    }
  }
}

}  // namespace osx
