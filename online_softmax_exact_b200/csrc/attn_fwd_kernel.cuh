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
//   * one CTA per SM (persistent), work unit = 256 query rows of one (batch, head) of
//     one (query chunk, key/value chunk) pair, held as two 128-row tiles in ping-pong:
//     the tensor core works on one tile while the other tile's softmax runs; a launch
//     carries up to kMaxPairs pairs, their units in one static schedule;
//   * warp 8 issues TMA loads (Q tiles once per unit, K and V tiles through rings of
//     shared-memory stages, 128-byte swizzle);
//   * warp 9 owns tensor memory and issues tcgen05.mma (from lane 0 at D = 128; at
//     D = 64 the whole warp runs the role in step and an elected lane issues):
//     S_t = Q_t K_j^T (both operands in shared memory) into TMEM, then O_t += P_t V_j
//     with P_t read from TMEM (written there by the softmax warps over S_t's columns);
//   * two softmax warpgroups: warpgroup t owns Q tile t, one thread per query row (TMEM
//     lane = row), all 128 keys of each key tile. A thread reads its 128 scores with
//     tcgen05.ld, reduces the tile maximum, and only then exponentiates (ex2, and at
//     d = 64 part of the values through an FMA-pipe polynomial), sums, packs P to bf16
//     and writes it back with tcgen05.st. The exponent base is the running maximum m,
//     moved only when a tile maximum exceeds it by more than 8 (log2 units); exactness
//     is kept because numerator and denominator share the same base. When m moves, the
//     thread rescales its row of O in TMEM before releasing P;
//   * epilogue: O / l and LSE = (m + log2 l) ln 2, written as fp32 (at D = 128 through a
//     per-warp shared-memory buffer, so that stores cover whole 128-byte row segments);
//     in accumulate mode the result is first combined with the normalised partial
//     (O_acc, LSE_acc) already in o/lse by the log-sum-exp rule of the merge (weights
//     e^(LSE - max LSE)).
//
// TMEM columns (512 allocated): S_0 [0,128), S_1 [128,256), O_0 [256,256+D),
// O_1 [384,384+D). P_t (bf16 pairs, keys in order) overwrites S_t columns [0,64): a
// thread holds all its scores in registers before it stores any P.
//
// Keys of the parent that lie past a pair's chunk but inside the tensor maps (pairs of a
// batched launch) are read into the pair's last key tile. Their scores are masked, so
// their P is exactly 0; the matching V rows are zeroed in shared memory before the P.V
// MMA reads them, so that a non-finite value there cannot turn 0 * V into NaN.
//
// All mbarrier waits are bounded (see mbar_wait); on time-out the kernel records it in
// the device status word, waits (bounded) for the copies it issued to land and for its
// MMAs to complete, frees TMEM and returns.
#pragma once

#include "sm100_ptx.cuh"

namespace osx {

constexpr int kMaxPairs = 48;

// Limit of the final wait for in-flight copies (see the producer's drain).
constexpr unsigned long long kDrainLimitNs = 100000000ull;  // 100 ms

// One (query chunk, key/value chunk) pair of a launch.
struct PairDesc {
  float* o;                  // [BH][Nq][D] fp32
  float* lse;                // [BH][Nq] fp32
  long long q_off, kv_off;   // global positions of the chunks' first rows (causal test)
  int q_row0, kv_row0;       // tensor-map row of the chunks' first rows
  int Nq, Nkv;               // chunk lengths
  int uniform;               // every unit visits all key tiles (no causal truncation)
  // Uniform pairs that read the same key/value chunk with the same shapes form a group
  // (consecutive in the table): pairs group_first .. group_first + group_n - 1.
  int group_first, group_n;
};

struct FwdParams {
  unsigned* status;    // device status word
  int BH;              // B * Hq
  int Hq, Hkv, group;  // group = Hq / Hkv
  int causal;
  float scale_log2;    // scale * log2(e), >= 0
  int o_vec8;          // every O is 32-byte aligned: store rows with 256-bit stores
  int accumulate;      // o/lse hold a partial over other keys: fold this chunk into it
  int kv_rows;         // rows of the K/V tensor maps (reads at or past them give zeros)
  int n_pairs;
  int unit_end[kMaxPairs];  // units of pairs 0..i: sum of ceil(Nq / 256) * BH
  PairDesc pair[kMaxPairs];
};

// Pairs (bit i: pair i of every 16) of a thread's scores whose 2^x comes from the FMA
// pipe in unmasked tiles, per head dimension. Measured on B200 (attn_fwd, TFLOP/s): at
// D = 64, 6 pairs of 16 (37.5%, with the warp-wide MMA issue below) gain ~4% over 4
// pairs issued from one lane, 8 pairs lose 15%; at D = 128 any share loses (the
// polynomial's ~5 instructions per value, against 1, compete for issue slots with a
// softmax that shares its tile period with twice the tensor work).
#ifndef OSX_EMU_MASK_64
#define OSX_EMU_MASK_64 0x9249u
#endif
#ifndef OSX_EMU_MASK_128
#define OSX_EMU_MASK_128 0x0000u
#endif
// K and V ring depths: 3 + 3 stages at D = 64; 2 + 2 at D = 128 (a third K stage fits in
// shared memory but measured no gain)
#ifndef OSX_STAGES_64
#define OSX_STAGES_64 3
#endif
#ifndef OSX_KSTAGES_128
#define OSX_KSTAGES_128 2
#endif

template <int D>
struct FwdCfg {
  static constexpr int kBM = 128;                    // rows per Q tile
  static constexpr int kBN = 128;                    // keys per KV tile
  // K and V ring depths (K is needed a P.V earlier than V)
  static constexpr int kKStages = (D == 128) ? OSX_KSTAGES_128 : OSX_STAGES_64;
  static constexpr int kVStages = (D == 128) ? 2 : OSX_STAGES_64;
  static constexpr uint32_t kTileBytes = kBM * D * 2;  // one 128-row bf16 tile
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = 2 * kTileBytes;
  static constexpr uint32_t kVOff = kKOff + kKStages * kTileBytes;
  static constexpr uint32_t kBarOff = kVOff + kVStages * kTileBytes;
  // barriers: q_full, q_empty, k_full[S], k_empty[S], v_full[S], v_empty[S],
  // s_full[2], p_full[2], o_done[2], drain
  static constexpr int kNumBars = 2 + 2 * kKStages + 2 * kVStages + 6 + 1;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;
  // epilogue staging (D = 128, outside accumulate mode): 32 rows x 32 fp32 (4 KB) per
  // softmax warp, to turn each thread's row into coalesced 128-byte row segments.
  // Measured on B200: +3-4% on the 128k GQA workload at D = 128, level elsewhere; at
  // D = 64 it loses 5%, and the accumulating ring 4%, so those store each row from its
  // own thread.
  static constexpr bool kStagedEpilogue = (D == 128);
  static constexpr uint32_t kStageOff = (kMiscOff + 16 + 1023) / 1024 * 1024;
  static constexpr uint32_t kStageBytes = kStagedEpilogue ? 8 * 4096 : 0;
  static constexpr uint32_t kSmemBytes = kStageOff + kStageBytes + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 232448, "shared memory per block");
  // warpgroups 0-1: softmax (tile t = warpgroup); warpgroup 2: {TMA producer, MMA
  // issuer, 2 idle}
  static constexpr int kThreads = 384;
  static constexpr int kSoftmaxWarps = 8;
  static constexpr int kWarpProducer = 8, kWarpMma = 9;
  // arrivals on a tile's p_full barrier: one per softmax warp of the tile
  static constexpr int kPFullCount = 4;
  // Registers per thread: 168 at launch (65536 / 384, rounded down to a multiple of 8);
  // after setmaxnreg the softmax warpgroups hold 216 and warpgroup 2 holds 72
  // (2 * 216 + 72 = 3 * 168, the launch's total: each SM sub-partition hosts one warp of
  // each warpgroup, so its 16K registers bound the sum). A softmax thread holds its
  // row's 128 scores in registers.
  static constexpr int kRegsSoftmax = 216;
  static constexpr int kRegsOther = 72;
  // pairs of each 32-score block whose 2^x comes from the FMA pipe (bit i: pair i)
  static constexpr uint32_t kEmu = (D == 64) ? OSX_EMU_MASK_64 : OSX_EMU_MASK_128;
  // MMA role run by the whole warp with elect.sync issue (D = 64), or by one lane
  // (D = 128). Warp-wide issue shortens each tile's P.V + Q.K^T chain; the softmax
  // warpgroups then overlap more, which at D = 128 costs more than the chain saves
  // (measured 1-3% slower there) and at D = 64 gains 2-4% with the larger FMA share.
  static constexpr bool kWarpIssue = (D == 64);
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 384;
};

__device__ __forceinline__ int unit_for_round(int round, int cta, int G) {
  // snake order: even rounds left to right, odd rounds right to left
  return round * G + ((round & 1) ? (G - 1 - cta) : cta);
}

// A work unit: 256 query rows (two 128-row tiles) of one (batch, head) of one pair.
// Units are numbered pair by pair (pairs in launch order, heaviest first). Within a
// group of pairs whose units all cost the same and that read one key/value chunk,
// heads are outermost (then pair, then row block), so that the CTAs running at one
// time share the key/value tiles of a few heads in L2; in other pairs row blocks go
// from the last to the first (heaviest first under the causal mask) with heads
// innermost, query heads sharing a key/value head side by side.
struct Unit {
  int pair, qp, bh;
  int n;  // key tiles the unit visits
};

__device__ __forceinline__ Unit decode_unit(const FwdParams& p, int u) {
  Unit un;
  int i = 0;
  while (i + 1 < p.n_pairs && u >= p.unit_end[i]) ++i;
  const PairDesc& pi = p.pair[i];
  const int n_qpairs = (pi.Nq + 255) / 256;  // the same for every pair of a group
  if (pi.uniform) {
    // heads outermost across the whole group, so that the CTAs running at one time
    // share the key/value tiles of a few heads in L2 for every query chunk at once
    const int first = pi.group_first;
    const int ug = u - (first ? p.unit_end[first - 1] : 0);
    const int per_head = pi.group_n * n_qpairs;
    un.bh = ug / per_head;
    const int rem = ug - un.bh * per_head;
    un.pair = first + rem / n_qpairs;
    un.qp = n_qpairs - 1 - rem % n_qpairs;
  } else {
    const int ul = u - (i ? p.unit_end[i - 1] : 0);
    un.pair = i;
    un.qp = n_qpairs - 1 - ul / p.BH;
    un.bh = ul % p.BH;
  }
  const PairDesc& pr = p.pair[un.pair];
  const int n_kv_tiles = (pr.Nkv + 127) / 128;
  // all key tiles, or under the causal mask those up to the last key visible to the
  // unit's last valid row; 0 means no row of the unit sees any key
  un.n = n_kv_tiles;
  if (p.causal) {
    long long last_row = (long long)un.qp * 256 + 255;
    if (last_row > pr.Nq - 1) last_row = pr.Nq - 1;
    const long long lim = pr.q_off + last_row - pr.kv_off;  // last visible key index
    if (lim < 0) {
      un.n = 0;
    } else {
      const long long n = lim / 128 + 1;
      if (n < n_kv_tiles) un.n = (int)n;
    }
  }
  return un;
}

// Row of the unit's last key tile from which the tile holds keys past the pair's chunk
// that the tensor maps still cover (so TMA loaded real data there rather than zeros);
// 128 when there are none.
__device__ __forceinline__ int tail_rows_to_zero(const FwdParams& p, const Unit& un) {
  const PairDesc& pr = p.pair[un.pair];
  const int end = un.n * 128;  // rows the unit's key tiles span, from the chunk start
  if (end <= pr.Nkv || pr.kv_row0 + pr.Nkv >= p.kv_rows) return 128;
  return pr.Nkv - (un.n - 1) * 128;
}

// Zero rows [r0, 128) of a K/V tile in shared memory (D/64 boxes of 128 rows x 128
// bytes; the 128-byte swizzle permutes 16-byte pieces within a row, so a row stays in
// its own 128 bytes), then make the writes visible to the tensor core's operand reads.
// kLanes threads (1, or the 32 lanes of a warp, `lane` each) share the stores.
template <int D, int kLanes>
__device__ __forceinline__ void zero_tile_rows(uint32_t tile, int r0, int lane) {
#pragma unroll 1
  for (int h = 0; h < D / 64; ++h) {
    const uint32_t end = tile + (h + 1) * 16384;
#pragma unroll 4
    for (uint32_t a = tile + h * 16384 + r0 * 128 + lane * 16; a < end; a += 16 * kLanes)
      st_shared_zero16(a);
  }
  fence_proxy_async_smem();
  if (kLanes == 32) __syncwarp();
}

// One thread per row: 32 of the row's scores -> 16 columns of bf16 P pairs at tP, against
// a known maximum (x = S * c - m); returns the sum of the 32 values of P. Masked elements
// (index > climit) get x = -inf, for which ex2 gives exactly 0.
template <bool kMasked, uint32_t kEmu>
__device__ __forceinline__ float softmax_row32(const uint32_t (&s)[32], uint32_t tP, float c,
                                               float m_use, int climit) {
  const uint64_t C2 = f2_pack(c, c);
  const uint64_t NM2 = f2_pack(-m_use, -m_use);
  uint64_t A01 = 0, A23 = 0;
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float x0, x1, e0, e1;
    const uint64_t X = f2_fma(f2_pack(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1])),
                              C2, NM2);
    uint64_t E;
    if (!kMasked && ((kEmu >> i) & 1u)) {
      E = exp2_poly_f32x2(X);
      f2_unpack(E, e0, e1);
    } else {
      f2_unpack(X, x0, x1);
      if (kMasked) {
        if (2 * i > climit) x0 = -INFINITY;
        if (2 * i + 1 > climit) x1 = -INFINITY;
      }
      e0 = ex2_approx(x0);
      e1 = ex2_approx(x1);
      E = f2_pack(e0, e1);
    }
    if (i & 1)
      A23 = f2_add(A23, E);
    else
      A01 = f2_add(A01, E);
    pk[i] = pack_bf16x2(e0, e1);
  }
  tmem_st16(tP, pk);
  float a0, a1, a2, a3;
  f2_unpack(A01, a0, a1);
  f2_unpack(A23, a2, a3);
  return (a0 + a1) + (a2 + a3);
}

template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::kThreads, 1)
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
  const int B_KF = 2, B_KE = 2 + C::kKStages, B_VF = 2 + 2 * C::kKStages,
            B_VE = 2 + 2 * C::kKStages + C::kVStages;
  const int B_SF = 2 + 2 * C::kKStages + 2 * C::kVStages, B_PF = B_SF + 2, B_OD = B_SF + 4,
            B_DRAIN = B_SF + 6;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(B_QF), 1);
    mbar_init(bar(B_QE), 1);
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(bar(B_KF + s), 1);
      mbar_init(bar(B_KE + s), 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(bar(B_VF + s), 1);
      mbar_init(bar(B_VE + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(B_SF + t), 1);
      mbar_init(bar(B_PF + t), C::kPFullCount);  // one arrival per softmax warp of the tile
      mbar_init(bar(B_OD + t), 1);
    }
    mbar_init(bar(B_DRAIN), 1);
    fence_mbar_init();
  }
  if (warp == C::kWarpMma) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == C::kWarpProducer && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int G = gridDim.x;
  const int n_units = p.unit_end[p.n_pairs - 1];

  if (warp >= C::kSoftmaxWarps) {
    regs_decrease<C::kRegsOther>();
    if (warp == C::kWarpProducer) {
      // ---------------------------------------------------------------- TMA producer
      if (lane == 0) {
        int ks = 0, kph = 0, vs = 0, vph = 0, qcount = 0;
        int k_arms = 0, v_arms = 0;  // K / V stage loads issued (for the final drain)
        bool ok = true;
        for (int r = 0; ok; ++r) {
          const int u = unit_for_round(r, blockIdx.x, G);
          if (u >= n_units) break;
          const Unit un = decode_unit(p, u);
          const int qp = un.qp, bh = un.bh, n = un.n;
          if (n == 0) continue;
          const PairDesc& pr = p.pair[un.pair];
          const int kvh = (bh / p.Hq) * p.Hkv + (bh % p.Hq) / p.group;
          // Q has one shared-memory buffer, so the next unit's Q can only be loaded once
          // this unit's last Q.K^T has read it; pull it into L2 now so that that load
          // is short.
          {
            const int u2 = unit_for_round(r + 1, blockIdx.x, G);
            if (u2 < n_units) {
              const Unit un2 = decode_unit(p, u2);
              if (un2.n > 0) {
                const PairDesc& pr2 = p.pair[un2.pair];
                for (int t = 0; t < 2; ++t)
                  for (int h = 0; h < D / 64; ++h)
                    tma_prefetch_l2_3d(&tmQ, h * 64, pr2.q_row0 + un2.qp * 256 + t * 128, un2.bh);
              }
            }
          }
          if (!(ok = mbar_wait(bar(B_QE), (qcount & 1) ^ 1, abort_flag, p.status))) break;
          ++qcount;
          mbar_arrive_expect_tx(bar(B_QF), 2 * C::kTileBytes);
          for (int t = 0; t < 2; ++t)
            for (int h = 0; h < D / 64; ++h)
              tma_load_3d(sbase + C::kQOff + t * C::kTileBytes + h * 16384, &tmQ, bar(B_QF),
                          h * 64, pr.q_row0 + qp * 256 + t * 128, bh);
          for (int j = 0; j < n; ++j) {
            if (!(ok = mbar_wait(bar(B_KE + ks), kph ^ 1, abort_flag, p.status))) break;
            mbar_arrive_expect_tx(bar(B_KF + ks), C::kTileBytes);
            for (int h = 0; h < D / 64; ++h)
              tma_load_3d(sbase + C::kKOff + ks * C::kTileBytes + h * 16384, &tmK, bar(B_KF + ks),
                          h * 64, pr.kv_row0 + j * 128, kvh);
            ++k_arms;
            if (++ks == C::kKStages) { ks = 0; kph ^= 1; }
            if (!(ok = mbar_wait(bar(B_VE + vs), vph ^ 1, abort_flag, p.status))) break;
            mbar_arrive_expect_tx(bar(B_VF + vs), C::kTileBytes);
            for (int h = 0; h < D / 64; ++h)
              tma_load_3d(sbase + C::kVOff + vs * C::kTileBytes + h * 16384, &tmV, bar(B_VF + vs),
                          h * 64, pr.kv_row0 + j * 128, kvh);
            ++v_arms;
            if (++vs == C::kVStages) { vs = 0; vph ^= 1; }
          }
        }
        // Wait until every copy issued has landed (the last armed phase of each full
        // barrier has completed), so that no copy writes shared memory after the CTA
        // exits. In a normal run they all have; after an abort some may still be in
        // flight. Bounded; if it runs out, wait a fixed time instead.
        bool drained = true;
        if (qcount > 0) drained &= mbar_wait_drain(bar(B_QF), (qcount - 1) & 1, kDrainLimitNs);
        for (int st = 0; st < C::kKStages; ++st) {
          const int kn = k_arms / C::kKStages + (st < k_arms % C::kKStages ? 1 : 0);
          if (kn > 0) drained &= mbar_wait_drain(bar(B_KF + st), (kn - 1) & 1, kDrainLimitNs);
        }
        for (int st = 0; st < C::kVStages; ++st) {
          const int vn = v_arms / C::kVStages + (st < v_arms % C::kVStages ? 1 : 0);
          if (vn > 0) drained &= mbar_wait_drain(bar(B_VF + st), (vn - 1) & 1, kDrainLimitNs);
        }
        if (!drained) {
          const unsigned long long t0 = globaltimer_ns();
          while (globaltimer_ns() - t0 < 200000ull) {
          }
        }
      }
    } else if (warp == C::kWarpMma) {
      // ---------------------------------------------------------------- MMA issuer
      // One lane, or the whole warp in step (every wait's outcome made uniform) with one
      // elected lane issuing each tcgen05 instruction.
      if (C::kWarpIssue || lane == 0) {
        constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
        int ks = 0, kph = 0, vs = 0, vph = 0, qcount = 0;
        int pv_steps = 0;  // P.V steps issued: both tiles' p_full barriers share its parity
        bool ok = true;
        auto wait_u = [&](uint32_t b, int parity, volatile int* af, unsigned* st) -> bool {
          const bool r = mbar_wait(b, parity, af, st);
          if constexpr (C::kWarpIssue) return __all_sync(0xffffffffu, r);
          return r;
        };
        auto commit = [&](uint32_t b) {
          if constexpr (C::kWarpIssue) mma_commit_warp(b); else mma_commit(b);
        };
        // Descriptors of the stage bases; the descriptor of (address + offset) is the
        // descriptor plus offset >> 4 (the start-address field is the low 14 bits and
        // every operand lies inside the CTA's shared memory window).
        const uint64_t dq0 = sdesc_sw128(sbase + C::kQOff, 16, 1024);
        const uint64_t dk0 = sdesc_sw128(sbase + C::kKOff, 16, 1024);
        const uint64_t dv0 = sdesc_sw128(sbase + C::kVOff, 16384, 1024);
        constexpr uint64_t kTileStep = C::kTileBytes >> 4;

        // O_t += P_t V (stage vstage); acc=false overwrites O_t. P_t's keys 0-127 sit in
        // S_t columns [0,64), 16 keys (8 columns) per MMA.
        auto issue_pv = [&](int t, int vstage, bool acc) {
          uint64_t dv = dv0 + (uint64_t)vstage * kTileStep;
          const uint32_t tO = tmem + (t ? C::kColO1 : C::kColO0);
          const uint32_t tP = tmem + (t ? C::kColS1 : C::kColS0);
          opaque(dv);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t b = dv + (uint64_t)(kk * 128);
            const uint32_t en = (acc || kk > 0) ? 1u : 0u;
            if constexpr (C::kWarpIssue)
              mma_ts_warp(tO, tP + kk * 8, b, idesc_pv, en);
            else
              mma_ts(tO, tP + kk * 8, b, idesc_pv, en);
          }
        };
        auto issue_qk = [&](int t, int kstage) {
          uint64_t dq = dq0 + (uint64_t)t * kTileStep;
          uint64_t dk = dk0 + (uint64_t)kstage * kTileStep;
          const uint32_t tS = tmem + (t ? C::kColS1 : C::kColS0);
          opaque(dq);
          opaque(dk);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)((kk / 4) * 1024 + (kk % 4) * 2);
            if constexpr (C::kWarpIssue)
              mma_ss_warp(tS, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
            else
              mma_ss(tS, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
          }
        };

        for (int r = 0; ok; ++r) {
          const int u = unit_for_round(r, blockIdx.x, G);
          if (u >= n_units) break;
          const Unit un = decode_unit(p, u);
          const int n = un.n;
          if (n == 0) continue;
          // V rows of the last key tile to zero before its P.V (the last of the unit)
          // reads them (128: none)
          const int vz_row = tail_rows_to_zero(p, un);
          if (!(ok = wait_u(bar(B_QF), qcount & 1, abort_flag, p.status))) break;
          ++qcount;
          tc_fence_after();
          for (int j = 0; j < n && ok; ++j) {
            if (!(ok = wait_u(bar(B_KF + ks), kph, abort_flag, p.status))) break;
            tc_fence_after();
            for (int t = 0; t < 2; ++t) {
              if (j > 0) {
                if (t == 0) {
                  if (!(ok = wait_u(bar(B_VF + vs), vph, abort_flag, p.status))) break;
                }
                if (!(ok = wait_u(bar(B_PF + t), pv_steps & 1, abort_flag, p.status))) break;
                tc_fence_after();
                issue_pv(t, vs, j > 1);
                if (t == 1) {
                  ++pv_steps;
                  commit(bar(B_VE + vs));
                  if (++vs == C::kVStages) { vs = 0; vph ^= 1; }
                }
              }
              issue_qk(t, ks);
              commit(bar(B_SF + t));
            }
            if (!ok) break;
            commit(bar(B_KE + ks));
            if (++ks == C::kKStages) { ks = 0; kph ^= 1; }
          }
          if (!ok) break;
          commit(bar(B_QE));
          // last P.V of the unit
          if (!(ok = wait_u(bar(B_VF + vs), vph, abort_flag, p.status))) break;
          if (vz_row < 128)
            zero_tile_rows<D, C::kWarpIssue ? 32 : 1>(sbase + C::kVOff + vs * C::kTileBytes,
                                                      vz_row, C::kWarpIssue ? lane : 0);
          for (int t = 0; t < 2; ++t) {
            if (!(ok = wait_u(bar(B_PF + t), pv_steps & 1, abort_flag, p.status))) break;
            tc_fence_after();
            issue_pv(t, vs, n > 1);
            commit(bar(B_OD + t));
          }
          if (!ok) break;
          ++pv_steps;
          commit(bar(B_VE + vs));
          if (++vs == C::kVStages) { vs = 0; vph ^= 1; }
        }
      }
    }
  } else {
    regs_increase<C::kRegsSoftmax>();
    // ------------------------------------------------------------------ softmax
    // one thread per row: thread r of softmax warpgroup t owns row r of Q tile t (TMEM
    // lane r) and all 128 keys of each key tile; the tile maximum is known before any
    // exponential, so P is computed once against the final base
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
      if (u >= n_units) break;
      const Unit un = decode_unit(p, u);
      const int qp = un.qp, bh = un.bh, n = un.n;
      const PairDesc& pr = p.pair[un.pair];
      const long long row0 = (long long)qp * 256 + t * 128;  // first row of this tile
      const long long row = row0 + r;
      const bool row_valid = row < pr.Nq;
      auto orow_of = [&]() { return pr.o + ((long long)bh * pr.Nq + row) * D; };
      auto lse_of = [&]() { return pr.lse + (long long)bh * pr.Nq + row; };

      if (n == 0) {
        // no key of this chunk is visible to the unit: the result is empty (O = 0,
        // LSE = -inf), and folding an empty result into an accumulator changes nothing
        if (row_valid && !p.accumulate) {
          float4* o4 = reinterpret_cast<float4*>(orow_of());
          for (int i = 0; i < D / 4; ++i) o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
          *lse_of() = -INFINITY;
        }
        continue;
      }

      // last visible key index for this row and for the tile's first row (both in
      // [-1, Nkv - 1])
      int lim_row = pr.Nkv - 1, lim_tile = pr.Nkv - 1;
      if (p.causal) {
        const long long a = pr.q_off + row - pr.kv_off, b = pr.q_off + row0 - pr.kv_off;
        lim_row = a < lim_row ? (a < -1 ? -1 : (int)a) : lim_row;
        lim_tile = b < lim_tile ? (b < -1 ? -1 : (int)b) : lim_tile;
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
        for (int q = 0; q < 4; ++q) tmem_ld32(tS + 32 * q, s[q]);
        tmem_ld_wait(s[0]);
        reg_fence(s[1]);
        reg_fence(s[2]);
        reg_fence(s[3]);

        // the same for every row of the tile (it depends on the tile's first row)
        const bool need_mask = (j * 128 + 127 > lim_tile);
        const int cl = lim_row - j * 128;  // keys with local index <= climit are visible
        const int climit = cl < -1 ? -1 : (cl > 127 ? 127 : cl);

        // tile maximum of the raw scores over the visible keys (four partial maxima);
        // two separate loops, so that unmasked tiles carry no per-element selects
        float mxa[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (need_mask) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float v0 =
                  (32 * q + 2 * i > climit) ? -INFINITY : __uint_as_float(s[q][2 * i]);
              const float v1 =
                  (32 * q + 2 * i + 1 > climit) ? -INFINITY : __uint_as_float(s[q][2 * i + 1]);
              float& acc = mxa[(q & 1) * 2 + (i & 1)];
              acc = fmax3(acc, v0, v1);
            }
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float& acc = mxa[(q & 1) * 2 + (i & 1)];
              acc = fmax3(acc, __uint_as_float(s[q][2 * i]), __uint_as_float(s[q][2 * i + 1]));
            }
        }
        const float mx = fmaxf(fmaxf(mxa[0], mxa[1]), fmaxf(mxa[2], mxa[3]));
        // The exponent base moves only when the tile maximum exceeds it by more than 8
        // (log2 units), and then to the tile maximum: numerator and denominator share the
        // base, so a stale one is exact, and P <= 2^8 stays well inside bf16 / fp32.
        const float m_tile = (mx == -INFINITY) ? -INFINITY : mx * c;
        const float m_new = (m_tile > m + 8.0f) ? m_tile : m;
        // 1 when unchanged (also when both are -inf), 0 when m was -inf
        const float alpha = (m_new == m) ? 1.f : ex2_approx(m - m_new);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;

        // P over S's first 64 columns (32 keys -> 16 columns): every score is in
        // registers already
        float sum;
        if (need_mask) {
          sum = softmax_row32<true, 0u>(s[0], tS, c, m_use, climit);
          sum += softmax_row32<true, 0u>(s[1], tS + 16, c, m_use, climit - 32);
          sum += softmax_row32<true, 0u>(s[2], tS + 32, c, m_use, climit - 64);
          sum += softmax_row32<true, 0u>(s[3], tS + 48, c, m_use, climit - 96);
        } else {
          sum = softmax_row32<false, C::kEmu>(s[0], tS, c, m_use, 127);
          sum += softmax_row32<false, C::kEmu>(s[1], tS + 16, c, m_use, 127);
          sum += softmax_row32<false, C::kEmu>(s[2], tS + 32, c, m_use, 127);
          sum += softmax_row32<false, C::kEmu>(s[3], tS + 48, c, m_use, 127);
        }
        l = l * alpha + sum;

        // rescale this row of O when its base moved (P.V of the previous key tile has
        // completed: the Q.K^T commit that released S follows it)
        const bool moved = (m_new != m) && (j > 0);
        if (__any_sync(0xffffffffu, moved)) {
          const float a = moved ? alpha : 1.f;
#pragma unroll 1
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
      float lse_acc = -INFINITY;
      float* lse_row = lse_of();
      if (p.accumulate && row_valid) lse_acc = *lse_row;
      const bool nonempty = l > 0.f;
      float lse_new = -INFINITY;
      if (nonempty) {
        float lg;
        asm("lg2.approx.f32 %0, %1;" : "=f"(lg) : "f"(l));
        lse_new = (m + lg) * 0.69314718055994530942f;
      }
      // out = a * O_acc + b * O_tmem
      float a = 0.f, b = nonempty ? 1.f / l : 0.f, lse_out = lse_new;
      if (p.accumulate) {
        const float M = fmaxf(lse_acc, lse_new);
        if (M == -INFINITY) {
          b = 0.f;
        } else {
          constexpr float kLog2e = 1.4426950408889634f;
          const float wa = ex2_approx((lse_acc - M) * kLog2e);  // 0 for an empty accumulator
          const float wn = ex2_approx((lse_new - M) * kLog2e);
          const float inv = 1.f / (wa + wn);
          a = wa * inv;
          b = nonempty ? wn * inv / l : 0.f;
          float lg;
          asm("lg2.approx.f32 %0, %1;" : "=f"(lg) : "f"(wa + wn));
          lse_out = M + lg * 0.69314718055994530942f;
        }
      }
      if (C::kStagedEpilogue && !p.accumulate) {
        // O in chunks of 32 columns: each thread scales its row's chunk and writes it to
        // the warp's staging buffer (16-byte pieces XOR-swizzled by row, so that neither
        // the row-wise writes nor the segment-wise reads conflict on banks); the warp then
        // stores 4 rows' 128-byte segments per instruction (one thread per row would
        // touch 32 lines per instruction). Accumulate mode, which also reads the old
        // values, keeps one thread per row (measured faster there).
        float4* stage = reinterpret_cast<float4*>(smem + C::kStageOff + warp * 4096);
        const int ch = lane & 7;
#pragma unroll 1
        for (int q4 = 0; q4 < D / 32; ++q4) {
          uint32_t ov[32];
          tmem_ld32(tO + q4 * 32, ov);
          tmem_ld_wait(ov);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            stage[lane * 8 + (c ^ (lane & 7))] =
                make_float4(__uint_as_float(ov[4 * c]) * b, __uint_as_float(ov[4 * c + 1]) * b,
                            __uint_as_float(ov[4 * c + 2]) * b, __uint_as_float(ov[4 * c + 3]) * b);
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int rl = i * 4 + (lane >> 3);  // row within the warp's 32
            const float4 v = stage[rl * 8 + (ch ^ (rl & 7))];
            const long long grow = row0 + wq * 32 + rl;
            if (grow < pr.Nq)
              *reinterpret_cast<float4*>(pr.o + ((long long)bh * pr.Nq + grow) * D + q4 * 32 +
                                         ch * 4) = v;
          }
          __syncwarp();  // the buffer is rewritten by the next chunk
        }
      } else {
        // one thread per row: 32-byte stores of the row's own chunk
#pragma unroll 1
        for (int q4 = 0; q4 < D / 32; ++q4) {
          uint32_t ov[32];
          tmem_ld32(tO + q4 * 32, ov);
          tmem_ld_wait(ov);
          if (row_valid) {
            float* dst = orow_of() + q4 * 32;
            float res[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) res[i] = __uint_as_float(ov[i]) * b;
            if (a != 0.f) {  // only then is the old accumulator read
#pragma unroll
              for (int i = 0; i < 32; i += 4) {
                const float4 old = *reinterpret_cast<const float4*>(dst + i);
                res[i] = fmaf(a, old.x, res[i]);
                res[i + 1] = fmaf(a, old.y, res[i + 1]);
                res[i + 2] = fmaf(a, old.z, res[i + 2]);
                res[i + 3] = fmaf(a, old.w, res[i + 3]);
              }
            }
            if (p.o_vec8) {
#pragma unroll
              for (int i = 0; i < 4; ++i)
                st_global_v8(dst + 8 * i, res[8 * i], res[8 * i + 1], res[8 * i + 2],
                             res[8 * i + 3], res[8 * i + 4], res[8 * i + 5], res[8 * i + 6],
                             res[8 * i + 7]);
            } else {
              float4* o4 = reinterpret_cast<float4*>(dst);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                o4[i] = make_float4(res[4 * i], res[4 * i + 1], res[4 * i + 2], res[4 * i + 3]);
            }
          }
        }
      }
      if (row_valid) *lse_row = lse_out;
      tc_fence_before();
    }
  }

  // ---------------------------------------------------------------------- teardown
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // let in-flight tensor-core work complete before TMEM is freed (the producer has
    // already waited for its copies)
    if (warp == C::kWarpMma && (C::kWarpIssue || lane == 0)) {
      // the commit comes from the issuer of the MMAs (the whole warp or lane 0)
      if constexpr (C::kWarpIssue)
        mma_commit_warp(bar(B_DRAIN));
      else
        mma_commit(bar(B_DRAIN));
      mbar_wait_drain(bar(B_DRAIN), 0, kDrainLimitNs);
    }
    __syncthreads();
  }
  if (warp == C::kWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace osx
