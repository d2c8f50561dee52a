// attn_fwd_kernel.cuh - exact blockwise attention forward for sm_100a.
//
// The method ("FlashAttention by hand", paragraphs on fused tiled attention, the
// running statistics, rescaling and the final division): for a block of query rows,
// stream key/value tiles through on-chip memory; for each tile form the logits, the
// tile maximum and the exponentials, fold them into a running maximum m and running
// denominator l, rescale the partial output when m grows, add P.V; divide once at the
// end. Scores never leave the SM.
//
// B200 mapping (our design, not the page's):
//   * one CTA per SM (persistent), work unit = 256 query rows of one (batch, head),
//     held as two 128-row tiles that two softmax warpgroups process in ping-pong, so
//     the tensor core works on one tile while the other tile's softmax runs;
//   * warp 8 issues TMA loads (Q tiles once per unit, K and V tiles through a ring of
//     shared-memory stages, 128-byte swizzle);
//   * warp 9 owns tensor memory and issues tcgen05.mma from one thread:
//     S_t = Q_t K_j^T (both operands in shared memory) into TMEM, then O_t += P_t V_j
//     with P_t read from TMEM (written there by the softmax warps over S_t's columns);
//   * softmax warpgroup t: thread r owns query row r of tile t (TMEM lane r), reads its
//     128 scores with tcgen05.ld, masks, takes the row maximum, exponentiates with
//     ex2, sums, packs P to bf16 and writes it back with tcgen05.st. The maximum used
//     for the exponent is only moved when the tile maximum exceeds it by more than
//     2^8 (exactness is kept because the same stale maximum is used for numerator and
//     denominator); when it moves, the warp rescales its rows of O in TMEM;
//   * epilogue: O / l and LSE = (m + log2 l) ln 2, written as fp32.
//
// TMEM columns (512 allocated): S_0 [0,128), S_1 [128,256), O_0 [256,256+D),
// O_1 [384,384+D). P_t (bf16 pairs) overwrites S_t columns [0,64) after S_t is read.
//
// All mbarrier waits are bounded (see mbar_wait); on time-out the kernel records it in
// the device status word, lets in-flight work drain, frees TMEM and returns.
#pragma once

#include "sm100_ptx.cuh"

namespace osx {

struct FwdParams {
  float* o;            // [BH][Nq][D] fp32
  float* lse;          // [BH][Nq] fp32
  unsigned* status;    // device status word
  long long Nq, Nkv;   // chunk lengths
  long long q_off, kv_off;
  int BH;              // B * Hq
  int Hq, Hkv, group;  // group = Hq / Hkv
  int causal;
  float scale_log2;    // scale * log2(e), >= 0
  int n_qpairs;        // ceil(Nq / 256)
  int n_units;         // n_qpairs * BH
  int n_kv_tiles;      // ceil(Nkv / 128)
  int o_vec8;          // O is 32-byte aligned: store rows with 256-bit stores
};

template <int D>
struct FwdCfg {
  static constexpr int kBM = 128;                    // rows per Q tile
  static constexpr int kBN = 128;                    // keys per KV tile
  static constexpr int kStages = (D == 128) ? 2 : 3; // K and V ring depth
  static constexpr uint32_t kTileBytes = kBM * D * 2;  // one 128-row bf16 tile
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = 2 * kTileBytes;
  static constexpr uint32_t kVOff = kKOff + kStages * kTileBytes;
  static constexpr uint32_t kBarOff = kVOff + kStages * kTileBytes;
  // barriers: q_full, q_empty, k_full[S], k_empty[S], v_full[S], v_empty[S],
  // s_full[2], p_full[2], o_done[2], drain
  static constexpr int kNumBars = 2 + 4 * kStages + 6 + 1;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;
  static constexpr uint32_t kSmemBytes = kMiscOff + 16 + 1024;  // + alignment slack
  // warpgroups: 0 and 1 softmax (Q tiles 0 and 1), 2 = {TMA producer, MMA issuer, 2 idle}
  static constexpr int kThreads = 384;
  // registers per thread: 168 at launch for all (each SM sub-partition hosts one warp
  // of each warpgroup); after setmaxnreg the softmax warpgroups hold 216 and warpgroup 2
  // holds 72 (216 + 216 + 72 = 3 * 168, the launch's total)
  static constexpr int kRegsSoftmax = 216;
  static constexpr int kRegsOther = 72;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 384;
};

__device__ __forceinline__ int unit_for_round(int round, int cta, int G) {
  // snake order: even rounds left to right, odd rounds right to left
  return round * G + ((round & 1) ? (G - 1 - cta) : cta);
}

// Number of key tiles a unit visits: all of them, or under the causal mask those up to
// the last key visible to the unit's last valid row. 0 means no row sees any key.
__device__ __forceinline__ int unit_kv_tiles(const FwdParams& p, int qp) {
  if (!p.causal) return p.n_kv_tiles;
  long long last_row = (long long)qp * 256 + 255;
  if (last_row > p.Nq - 1) last_row = p.Nq - 1;
  const long long lim = p.q_off + last_row - p.kv_off;  // last visible key index
  if (lim < 0) return 0;
  const long long n = lim / 128 + 1;
  return n < p.n_kv_tiles ? (int)n : p.n_kv_tiles;
}

// One row's P for one 128-key tile: x = S * scale*log2(e) - m (packed pairs), P = 2^x,
// written back to TMEM as bf16 pairs over the first 64 columns of S; returns sum(P).
// Masked tiles send every element through ex2 (so that -inf gives exactly 0); other
// tiles send 4 of every 16 pairs through the FMA-pipe polynomial to share the load with
// the exp unit.
template <bool kMasked>
__device__ __forceinline__ float softmax_tile(uint32_t (&s)[4][32], uint32_t tS, float c,
                                              float m_use, int climit) {
  const uint64_t C2 = f2_pack(c, c);
  const uint64_t NM2 = f2_pack(-m_use, -m_use);
  uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = f2_pack(0.f, 0.f);
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint64_t X = f2_fma(f2_pack(__uint_as_float(s[q4][2 * i]),
                                        __uint_as_float(s[q4][2 * i + 1])), C2, NM2);
      float x0, x1, e0, e1;
      f2_unpack(X, x0, x1);
      if (kMasked) {
        if (q4 * 32 + 2 * i > climit) x0 = -INFINITY;
        if (q4 * 32 + 2 * i + 1 > climit) x1 = -INFINITY;
        e0 = ex2_approx(x0);
        e1 = ex2_approx(x1);
      } else if (i >= 12) {
        exp2_poly_pair(x0, x1, e0, e1);
      } else {
        e0 = ex2_approx(x0);
        e1 = ex2_approx(x1);
      }
      if (i & 1)
        acc1 = f2_add(acc1, f2_pack(e0, e1));
      else
        acc0 = f2_add(acc0, f2_pack(e0, e1));
      pk[i] = pack_bf16x2(e0, e1);
    }
    tmem_st16(tS + q4 * 16, pk);
  }
  float a, b, cc, d;
  f2_unpack(acc0, a, b);
  f2_unpack(acc1, cc, d);
  return (a + b) + (cc + d);
}

template <int D>
__global__ void __launch_bounds__(384, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int B_QF = 0, B_QE = 1;
  const int B_KF = 2, B_KE = 2 + C::kStages, B_VF = 2 + 2 * C::kStages,
            B_VE = 2 + 3 * C::kStages;
  const int B_SF = 2 + 4 * C::kStages, B_PF = B_SF + 2, B_OD = B_SF + 4, B_DRAIN = B_SF + 6;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(B_QF), 1);
    mbar_init(bar(B_QE), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(B_KF + s), 1);
      mbar_init(bar(B_KE + s), 1);
      mbar_init(bar(B_VF + s), 1);
      mbar_init(bar(B_VE + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(B_SF + t), 1);
      mbar_init(bar(B_PF + t), 4);  // one arrival per softmax warp
      mbar_init(bar(B_OD + t), 1);
    }
    mbar_init(bar(B_DRAIN), 1);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int G = gridDim.x;

  if (warp >= 8) {
  regs_decrease<C::kRegsOther>();
  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int ks = 0, kph = 0, vs = 0, vph = 0, qcount = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int u = unit_for_round(r, blockIdx.x, G);
        if (u >= p.n_units) break;
        const int qp = p.n_qpairs - 1 - u / p.BH;
        const int bh = u % p.BH;
        const int n = unit_kv_tiles(p, qp);
        if (n == 0) continue;
        const int kvh = (bh / p.Hq) * p.Hkv + (bh % p.Hq) / p.group;
        if (!(ok = mbar_wait(bar(B_QE), (qcount & 1) ^ 1, abort_flag, p.status))) break;
        ++qcount;
        mbar_arrive_expect_tx(bar(B_QF), 2 * C::kTileBytes);
        for (int t = 0; t < 2; ++t)
          for (int h = 0; h < D / 64; ++h)
            tma_load_3d(sbase + C::kQOff + t * C::kTileBytes + h * 16384, &tmQ, bar(B_QF), h * 64,
                        qp * 256 + t * 128, bh);
        for (int j = 0; j < n; ++j) {
          if (!(ok = mbar_wait(bar(B_KE + ks), kph ^ 1, abort_flag, p.status))) break;
          mbar_arrive_expect_tx(bar(B_KF + ks), C::kTileBytes);
          for (int h = 0; h < D / 64; ++h)
            tma_load_3d(sbase + C::kKOff + ks * C::kTileBytes + h * 16384, &tmK, bar(B_KF + ks),
                        h * 64, j * 128, kvh);
          if (++ks == C::kStages) { ks = 0; kph ^= 1; }
          if (!(ok = mbar_wait(bar(B_VE + vs), vph ^ 1, abort_flag, p.status))) break;
          mbar_arrive_expect_tx(bar(B_VF + vs), C::kTileBytes);
          for (int h = 0; h < D / 64; ++h)
            tma_load_3d(sbase + C::kVOff + vs * C::kTileBytes + h * 16384, &tmV, bar(B_VF + vs),
                        h * 64, j * 128, kvh);
          if (++vs == C::kStages) { vs = 0; vph ^= 1; }
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      int ks = 0, kph = 0, vs = 0, vph = 0, qcount = 0;
      int pcount[2] = {0, 0};
      bool ok = true;

      // O_t += P_t V (stage vstage); acc=false overwrites O_t
      auto issue_pv = [&](int t, int vstage, bool acc) {
        const uint32_t vaddr = sbase + C::kVOff + vstage * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + (t ? C::kColO1 : C::kColO0), tmem + (t ? C::kColS1 : C::kColS0) + kk * 8, sdesc_sw128(vaddr + kk * 2048, 16384, 1024),
                 idesc_pv, (acc || kk > 0) ? 1u : 0u);
      };
      auto issue_qk = [&](int t, int kstage) {
        const uint32_t qaddr = sbase + C::kQOff + t * C::kTileBytes;
        const uint32_t kaddr = sbase + C::kKOff + kstage * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
          mma_ss(tmem + (t ? C::kColS1 : C::kColS0), sdesc_sw128(qaddr + off, 16, 1024),
                 sdesc_sw128(kaddr + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
      };

      for (int r = 0; ok; ++r) {
        const int u = unit_for_round(r, blockIdx.x, G);
        if (u >= p.n_units) break;
        const int qp = p.n_qpairs - 1 - u / p.BH;
        const int n = unit_kv_tiles(p, qp);
        if (n == 0) continue;
        if (!(ok = mbar_wait(bar(B_QF), qcount & 1, abort_flag, p.status))) break;
        ++qcount;
        tc_fence_after();
        for (int j = 0; j < n && ok; ++j) {
          if (!(ok = mbar_wait(bar(B_KF + ks), kph, abort_flag, p.status))) break;
          tc_fence_after();
          for (int t = 0; t < 2; ++t) {
            if (j > 0) {
              if (t == 0) {
                if (!(ok = mbar_wait(bar(B_VF + vs), vph, abort_flag, p.status))) break;
              }
              if (!(ok = mbar_wait(bar(B_PF + t), pcount[t] & 1, abort_flag, p.status))) break;
              ++pcount[t];
              tc_fence_after();
              issue_pv(t, vs, j > 1);
              if (t == 1) {
                mma_commit(bar(B_VE + vs));
                if (++vs == C::kStages) { vs = 0; vph ^= 1; }
              }
            }
            issue_qk(t, ks);
            mma_commit(bar(B_SF + t));
          }
          if (!ok) break;
          mma_commit(bar(B_KE + ks));
          if (++ks == C::kStages) { ks = 0; kph ^= 1; }
        }
        if (!ok) break;
        mma_commit(bar(B_QE));
        // last P.V of the unit
        if (!(ok = mbar_wait(bar(B_VF + vs), vph, abort_flag, p.status))) break;
        for (int t = 0; t < 2; ++t) {
          if (!(ok = mbar_wait(bar(B_PF + t), pcount[t] & 1, abort_flag, p.status))) break;
          ++pcount[t];
          tc_fence_after();
          issue_pv(t, vs, n > 1);
          mma_commit(bar(B_OD + t));
        }
        if (!ok) break;
        mma_commit(bar(B_VE + vs));
        if (++vs == C::kStages) { vs = 0; vph ^= 1; }
      }
    }
  }
  } else {
    regs_increase<C::kRegsSoftmax>();
    // ------------------------------------------------------------------ softmax warpgroups
    const int t = warp / 4;                 // which Q tile of the unit
    const int wq = warp % 4;                // warp's TMEM lane quarter
    const int r = wq * 32 + lane;           // row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_base + (t ? C::kColS1 : C::kColS0);
    const uint32_t tO = tmem + lane_base + (t ? C::kColO1 : C::kColO0);
    const float c = p.scale_log2;
    int scount = 0, ocount = 0;
    bool ok = true;

    for (int rr = 0; ok; ++rr) {
      const int u = unit_for_round(rr, blockIdx.x, G);
      if (u >= p.n_units) break;
      const int qp = p.n_qpairs - 1 - u / p.BH;
      const int bh = u % p.BH;
      const int n = unit_kv_tiles(p, qp);
      const long long row0 = (long long)qp * 256 + t * 128;  // first row of this tile
      const long long row = row0 + r;
      const bool row_valid = row < p.Nq;
      float* orow = p.o + ((long long)bh * p.Nq + row) * D;

      if (n == 0) {
        if (row_valid) {
          float4* o4 = reinterpret_cast<float4*>(orow);
          for (int i = 0; i < D / 4; ++i) o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
          p.lse[(long long)bh * p.Nq + row] = -INFINITY;
        }
        continue;
      }

      // last visible key index for this row (local to the chunk), and for the tile's
      // first row (which decides whether a tile needs the per-element mask)
      long long lim_row = p.Nkv - 1, lim_tile = p.Nkv - 1;
      if (p.causal) {
        const long long a = p.q_off + row - p.kv_off, b = p.q_off + row0 - p.kv_off;
        lim_row = a < lim_row ? a : lim_row;
        lim_tile = b < lim_tile ? b : lim_tile;
      }

      float m = -INFINITY;  // running maximum (log2 units) used for the exponent
      float l = 0.f;        // running denominator

      for (int j = 0; j < n; ++j) {
        ok = mbar_wait(bar(B_SF + t), scount & 1, abort_flag, p.status);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++scount;
        tc_fence_after();

        uint32_t s[4][32];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(tS + q4 * 32, s[q4]);
        tmem_ld_wait(s[0]);
        reg_fence(s[1]);
        reg_fence(s[2]);
        reg_fence(s[3]);

        const long long kbase = (long long)j * 128;
        const bool need_mask = (kbase + 127 > lim_tile);
        // keys with local column <= climit are visible for this row
        long long cl = lim_row - kbase;
        const int climit = cl < -1 ? -1 : (cl > 127 ? 127 : (int)cl);

        if (need_mask) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (q4 * 32 + i > climit) s[q4][i] = __float_as_uint(-INFINITY);
        }
        float mx;
        {
          float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            m0 = fmax3(m0, __uint_as_float(s[0][2 * i]), __uint_as_float(s[0][2 * i + 1]));
            m1 = fmax3(m1, __uint_as_float(s[1][2 * i]), __uint_as_float(s[1][2 * i + 1]));
            m2 = fmax3(m2, __uint_as_float(s[2][2 * i]), __uint_as_float(s[2][2 * i + 1]));
            m3 = fmax3(m3, __uint_as_float(s[3][2 * i]), __uint_as_float(s[3][2 * i + 1]));
          }
          mx = fmax3(m0, m1, fmaxf(m2, m3));
        }
        const float m_tile = (mx == -INFINITY) ? -INFINITY : mx * c;
        const float m_new = (m_tile > m + 8.0f) ? m_tile : m;
        // 1 when unchanged (also when both are -inf), 0 when m was -inf
        const float alpha = (m_new == m) ? 1.f : ex2_approx(m - m_new);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;

        float sum = need_mask ? softmax_tile<true>(s, tS, c, m_use, climit)
                              : softmax_tile<false>(s, tS, c, m_use, climit);
        l = l * alpha + sum;

        // rescale this warp's rows of O when any of them moved its maximum
        const bool moved = (m_new != m) && (j > 0);
        if (__any_sync(0xffffffffu, moved)) {
          const float a = moved ? alpha : 1.f;
#pragma unroll
          for (int q4 = 0; q4 < D / 32; ++q4) {
            uint32_t ov[32];
            tmem_ld32(tO + q4 * 32, ov);
            tmem_ld_wait(ov);
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * a);
            tmem_st32(tO + q4 * 32, ov);
          }
        }
        m = m_new;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_PF + t));
      }
      if (!ok) break;

      // ---------------------------------------------------------------- epilogue
      ok = mbar_wait(bar(B_OD + t), ocount & 1, abort_flag, p.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ++ocount;
      tc_fence_after();
      const bool nonempty = l > 0.f;
      const float inv_l = nonempty ? 1.f / l : 0.f;
#pragma unroll
      for (int q4 = 0; q4 < D / 32; ++q4) {
        uint32_t ov[32];
        tmem_ld32(tO + q4 * 32, ov);
        tmem_ld_wait(ov);
        if (row_valid) {
          float* dst = orow + q4 * 32;
          if (p.o_vec8) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              st_global_v8(dst + 8 * i, __uint_as_float(ov[8 * i]) * inv_l,
                           __uint_as_float(ov[8 * i + 1]) * inv_l,
                           __uint_as_float(ov[8 * i + 2]) * inv_l,
                           __uint_as_float(ov[8 * i + 3]) * inv_l,
                           __uint_as_float(ov[8 * i + 4]) * inv_l,
                           __uint_as_float(ov[8 * i + 5]) * inv_l,
                           __uint_as_float(ov[8 * i + 6]) * inv_l,
                           __uint_as_float(ov[8 * i + 7]) * inv_l);
          } else {
            float4* o4 = reinterpret_cast<float4*>(dst);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              o4[i] = make_float4(__uint_as_float(ov[4 * i]) * inv_l,
                                  __uint_as_float(ov[4 * i + 1]) * inv_l,
                                  __uint_as_float(ov[4 * i + 2]) * inv_l,
                                  __uint_as_float(ov[4 * i + 3]) * inv_l);
          }
        }
      }
      if (row_valid) {
        float lse;
        if (nonempty) {
          float lg;
          asm("lg2.approx.f32 %0, %1;" : "=f"(lg) : "f"(l));
          lse = (m + lg) * 0.69314718055994530942f;
        } else {
          lse = -INFINITY;
        }
        p.lse[(long long)bh * p.Nq + row] = lse;
      }
      tc_fence_before();
    }
  }

  // ---------------------------------------------------------------------- teardown
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // let in-flight tensor-core work and copies land before TMEM is freed
    if (warp == 9 && lane == 0) {
      mma_commit(bar(B_DRAIN));
      volatile int dummy = 0;
      mbar_wait(bar(B_DRAIN), 0, &dummy, p.status);
    }
    if (warp == 8 && lane == 0) {
      const unsigned long long t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 200000ull) {
      }
    }
    __syncthreads();
  }
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace osx
