// attn_api.cpp - the C ABI of libattn: argument checks, fault injection for tests, and
// dispatch to the launchers. Every check here runs before any CUDA call, so invalid
// arguments are reported without touching a device.
#include <cmath>
#include <cstdint>
#include <vector>

#include "../../include/attn.h"
#include "attn_internal.h"

namespace {

int g_inject_status = ATTN_OK;
int g_inject_count = 0;

// Largest chunk length: TMA row coordinates are 32-bit and a unit reaches 256 rows past
// its start.
constexpr int64_t kMaxRows = (int64_t(1) << 31) - 512;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Span {
  uintptr_t lo, hi;  // [lo, hi)
};

Span span(const void* p, uint64_t bytes) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  return Span{lo, lo + static_cast<uintptr_t>(bytes)};
}

bool overlap(Span a, Span b) { return a.lo < b.hi && b.lo < a.hi; }

attn_status_t take_injected() {
  if (g_inject_count > 0) {
    --g_inject_count;
    return static_cast<attn_status_t>(g_inject_status);
  }
  return ATTN_OK;
}

attn_status_t check_and_launch(const void* q, const void* k, const void* v, float* o, float* lse,
                               int B, int Hq, int Hkv, int64_t Nq, int64_t Nkv, int64_t q_ld,
                               int64_t kv_ld, int64_t q_off, int64_t kv_off, int d, int causal,
                               float scale, void* stream, int accumulate) {
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (Nq < 1 || Nkv < 1 || q_ld < Nq || kv_ld < Nkv || q_off < 0 || kv_off < 0)
    return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (Nq > kMaxRows || Nkv > kMaxRows || q_ld > kMaxRows || kv_ld > kMaxRows)
    return ATTN_ERR_UNSUPPORTED;
  if ((int64_t)B * Hq > (int64_t(1) << 30) || q_off > (int64_t(1) << 60) ||
      kv_off > (int64_t(1) << 60))
    return ATTN_ERR_UNSUPPORTED;

  const uint64_t bh = (uint64_t)B * Hq, bhkv = (uint64_t)B * Hkv;
  const Span sq = span(q, ((bh - 1) * q_ld + Nq) * d * 2);
  const Span sk = span(k, ((bhkv - 1) * kv_ld + Nkv) * d * 2);
  const Span sv = span(v, ((bhkv - 1) * kv_ld + Nkv) * d * 2);
  const Span so = span(o, bh * Nq * d * 4);
  const Span sl = span(lse, bh * Nq * 4);
  if (overlap(so, sq) || overlap(so, sk) || overlap(so, sv) || overlap(sl, sq) ||
      overlap(sl, sk) || overlap(sl, sv) || overlap(so, sl))
    return ATTN_ERR_INVALID_ARG;

  attn_status_t inj = take_injected();
  if (inj != ATTN_OK) return inj;

  // one pair; the tensor maps cover exactly the two chunks, so rows past a chunk read
  // as zero
  osx::PairLaunch pr{0, Nq, 0, Nkv, q_off, kv_off, o, lse};
  osx::FwdLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.q_rows = Nq;
  a.kv_rows = Nkv;
  a.q_ld = q_ld;
  a.kv_ld = kv_ld;
  a.d = d;
  a.causal = causal;
  a.scale = scale;
  a.accumulate = accumulate;
  a.n_pairs = 1;
  a.pairs = &pr;
  return static_cast<attn_status_t>(osx::launch_fwd(a, static_cast<cudaStream_t>(stream)));
}

// Cost of a pair's heaviest work unit (its last 256-row block under the causal mask), in
// key tiles: the batched launch orders pairs by it, heaviest first.
int64_t pair_heaviest_unit(const attn_pair_t& p, int causal) {
  const int64_t tiles = (p.kv_len + 127) / 128;
  if (!causal) return tiles;
  const int64_t lim = p.q_off + p.q_len - 1 - p.kv_off;
  if (lim < 0) return 0;
  const int64_t n = lim / 128 + 1;
  return n < tiles ? n : tiles;
}

// Whether all of a pair's work units cost the same: even its first 256-row block sees
// every key tile (the kernel's own test for its head-major unit order).
bool pair_uniform(const attn_pair_t& p, int causal) {
  const int64_t tiles = (p.kv_len + 127) / 128;
  const int64_t lim0 = p.q_off + (p.q_len < 256 ? p.q_len : 256) - 1 - p.kv_off;
  return !causal || lim0 >= (tiles - 1) * 128;
}

// Launch order of two pairs: heavier heaviest unit first; on a tie, pairs with equal
// units before pairs with a causal cut, so that the grid's last units are the cut
// pairs' light ones; among pairs with equal units, those that read the same key/value
// chunk side by side (the kernel then runs them head by head across the group).
bool goes_before(const attn_pair_t& a, const attn_pair_t& b, int causal) {
  const int64_t ca = pair_heaviest_unit(a, causal), cb = pair_heaviest_unit(b, causal);
  if (ca != cb) return ca > cb;
  const bool ua = pair_uniform(a, causal), ub = pair_uniform(b, causal);
  if (ua != ub) return ua;
  if (ua) {
    if (a.kv_start != b.kv_start) return a.kv_start < b.kv_start;
    if (a.kv_len != b.kv_len) return a.kv_len < b.kv_len;
    if (a.q_len != b.q_len) return a.q_len < b.q_len;
  }
  return false;
}

}  // namespace

extern "C" {

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ATTN_OK: success";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG: invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED: shape or size not supported";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA: a CUDA call failed";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT: a device-side wait ran out of time";
    case ATTN_ERR_INJECTED: return "ATTN_ERR_INJECTED: failure injected by attn_debug_inject";
    default: return "unknown attn status";
  }
}

int attn_version(void) { return (1 << 16) | 2; }

attn_status_t attn_fwd(const void* q, const void* k, const void* v, float* o, float* lse, int B,
                       int Hq, int Hkv, int64_t N, int d, int causal, float scale, void* stream) {
  return check_and_launch(q, k, v, o, lse, B, Hq, Hkv, N, N, N, N, 0, 0, d, causal, scale, stream,
                          0);
}

attn_status_t attn_fwd_partial(const void* q, const void* k_chunk, const void* v_chunk,
                               float* o_part, float* lse_part, int B, int Hq, int Hkv, int64_t Nq,
                               int64_t Nkv, int64_t q_ld, int64_t kv_ld, int64_t q_off,
                               int64_t kv_off, int d, int causal, float scale, void* stream) {
  return check_and_launch(q, k_chunk, v_chunk, o_part, lse_part, B, Hq, Hkv, Nq, Nkv, q_ld, kv_ld,
                          q_off, kv_off, d, causal, scale, stream, 0);
}

attn_status_t attn_fwd_partial_acc(const void* q, const void* k_chunk, const void* v_chunk,
                                   float* o_acc, float* lse_acc, int B, int Hq, int Hkv,
                                   int64_t Nq, int64_t Nkv, int64_t q_ld, int64_t kv_ld,
                                   int64_t q_off, int64_t kv_off, int d, int causal, float scale,
                                   void* stream) {
  return check_and_launch(q, k_chunk, v_chunk, o_acc, lse_acc, B, Hq, Hkv, Nq, Nkv, q_ld, kv_ld,
                          q_off, kv_off, d, causal, scale, stream, 1);
}

attn_status_t attn_merge(const float* const* o_parts, const float* const* lse_parts, int n_parts,
                         float* o, float* lse, int64_t rows, int d, void* stream) {
  if (!o_parts || !lse_parts || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (n_parts < 1 || rows < 1) return ATTN_ERR_INVALID_ARG;
  if (!aligned(o, 32) || !aligned(lse, 4)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (n_parts > ATTN_MAX_MERGE_PARTS) return ATTN_ERR_UNSUPPORTED;
  if (rows > (int64_t(1) << 40)) return ATTN_ERR_UNSUPPORTED;
  const Span so = span(o, (uint64_t)rows * d * 4);
  const Span sl = span(lse, (uint64_t)rows * 4);
  if (overlap(so, sl)) return ATTN_ERR_INVALID_ARG;
  for (int i = 0; i < n_parts; ++i) {
    if (!o_parts[i] || !lse_parts[i]) return ATTN_ERR_INVALID_ARG;
    if (!aligned(o_parts[i], 32) || !aligned(lse_parts[i], 4)) return ATTN_ERR_INVALID_ARG;
    const Span po = span(o_parts[i], (uint64_t)rows * d * 4);
    const Span pl = span(lse_parts[i], (uint64_t)rows * 4);
    if (overlap(so, po) || overlap(so, pl) || overlap(sl, po) || overlap(sl, pl))
      return ATTN_ERR_INVALID_ARG;
  }
  attn_status_t inj = take_injected();
  if (inj != ATTN_OK) return inj;
  return static_cast<attn_status_t>(osx::launch_merge(o_parts, lse_parts, n_parts, o, lse, rows, d,
                                                      static_cast<cudaStream_t>(stream)));
}

attn_status_t attn_device_status(void* stream, int reset) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  unsigned st = 0;
  if (osx::read_device_status(&st, reset) != ATTN_OK) return ATTN_ERR_CUDA;
  return st ? ATTN_ERR_TIMEOUT : ATTN_OK;
}

attn_status_t attn_debug_inject(int status, int count) {
  if (count < 0) return ATTN_ERR_INVALID_ARG;
  if (count > 0 && (status <= ATTN_OK || status > ATTN_ERR_INJECTED)) return ATTN_ERR_INVALID_ARG;
  g_inject_status = status;
  g_inject_count = count;
  return ATTN_OK;
}

attn_status_t attn_debug_wait_timeout(int64_t limit_cycles, void* stream) {
  if (limit_cycles < 1 || limit_cycles > (int64_t(1) << 31)) return ATTN_ERR_INVALID_ARG;
  return static_cast<attn_status_t>(
      osx::launch_wait_probe(limit_cycles, static_cast<cudaStream_t>(stream)));
}

attn_status_t attn_fwd_partial_batch(const void* q, const void* k, const void* v, int B, int Hq,
                                     int Hkv, int64_t q_ld, int64_t kv_ld, int d, int causal,
                                     float scale, const attn_pair_t* pairs, int n_pairs,
                                     int accumulate, void* stream) {
  if (!q || !k || !v || !pairs) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || q_ld < 1 || kv_ld < 1)
    return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (accumulate != 0 && accumulate != 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16)) return ATTN_ERR_INVALID_ARG;
  if (n_pairs < 1) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (n_pairs > ATTN_MAX_BATCH_PAIRS) return ATTN_ERR_UNSUPPORTED;
  if (q_ld > kMaxRows || kv_ld > kMaxRows || (int64_t)B * Hq > (int64_t(1) << 30))
    return ATTN_ERR_UNSUPPORTED;
  const uint64_t bh = (uint64_t)B * Hq, bhkv = (uint64_t)B * Hkv;
  const Span sq = span(q, bh * q_ld * d * 2);
  const Span sk = span(k, bhkv * kv_ld * d * 2);
  const Span sv = span(v, bhkv * kv_ld * d * 2);
  for (int i = 0; i < n_pairs; ++i) {
    const attn_pair_t& p = pairs[i];
    if (!p.o || !p.lse || !aligned(p.o, 16) || !aligned(p.lse, 4)) return ATTN_ERR_INVALID_ARG;
    if (p.q_start < 0 || p.q_len < 1 || p.q_start + p.q_len > q_ld || p.kv_start < 0 ||
        p.kv_len < 1 || p.kv_start + p.kv_len > kv_ld || p.q_off < 0 || p.kv_off < 0 ||
        p.q_off > (int64_t(1) << 60) || p.kv_off > (int64_t(1) << 60))
      return ATTN_ERR_INVALID_ARG;
    const Span so = span(p.o, bh * p.q_len * d * 4);
    const Span sl = span(p.lse, bh * p.q_len * 4);
    if (overlap(so, sq) || overlap(so, sk) || overlap(so, sv) || overlap(sl, sq) ||
        overlap(sl, sk) || overlap(sl, sv) || overlap(so, sl))
      return ATTN_ERR_INVALID_ARG;
    for (int j = 0; j < i; ++j) {  // no two pairs may write the same memory
      const Span po = span(pairs[j].o, bh * pairs[j].q_len * d * 4);
      const Span pl = span(pairs[j].lse, bh * pairs[j].q_len * 4);
      if (overlap(so, po) || overlap(so, pl) || overlap(sl, po) || overlap(sl, pl))
        return ATTN_ERR_INVALID_ARG;
    }
  }
  attn_status_t inj = take_injected();
  if (inj != ATTN_OK) return inj;

  // heaviest pairs first, so that the persistent grid's last units are the light ones
  int order[ATTN_MAX_BATCH_PAIRS];
  for (int i = 0; i < n_pairs; ++i) order[i] = i;
  for (int i = 1; i < n_pairs; ++i) {  // stable insertion sort, n_pairs <= 48
    const int x = order[i];
    int j = i - 1;
    while (j >= 0 && goes_before(pairs[x], pairs[order[j]], causal)) {
      order[j + 1] = order[j];
      --j;
    }
    order[j + 1] = x;
  }
  osx::PairLaunch pl[ATTN_MAX_BATCH_PAIRS];
  for (int i = 0; i < n_pairs; ++i) {
    const attn_pair_t& p = pairs[order[i]];
    pl[i] = osx::PairLaunch{p.q_start, p.q_len, p.kv_start, p.kv_len, p.q_off, p.kv_off, p.o,
                            p.lse};
  }
  osx::FwdLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.q_rows = q_ld;
  a.kv_rows = kv_ld;
  a.q_ld = q_ld;
  a.kv_ld = kv_ld;
  a.d = d;
  a.causal = causal;
  a.scale = scale;
  a.accumulate = accumulate;
  a.n_pairs = n_pairs;
  a.pairs = pl;
  return static_cast<attn_status_t>(osx::launch_fwd(a, static_cast<cudaStream_t>(stream)));
}

attn_status_t attn_ring_fwd_host(const void* q_h, const void* k_h, const void* v_h, float* o_h,
                                 float* lse_h, void* q_d, void* k_d, void* v_d, float* o_d,
                                 float* lse_d, float* ws_o, float* ws_lse, int ws_slots, int B,
                                 int Hq, int Hkv, int64_t N, int d, int n_chunks, int causal,
                                 float scale, void* stream, void* h2d_stream, void* d2h_stream) {
  if (!q_h || !k_h || !v_h || !o_h || !lse_h || !q_d || !k_d || !v_d || !o_d || !lse_d)
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || N < 1) return ATTN_ERR_INVALID_ARG;
  if (n_chunks < 1 || N % n_chunks != 0) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q_d, 16) || !aligned(k_d, 16) || !aligned(v_d, 16) || !aligned(o_d, 32) ||
      !aligned(lse_d, 4))
    return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (n_chunks > ATTN_MAX_BATCH_PAIRS) return ATTN_ERR_UNSUPPORTED;
  if (N > kMaxRows || (int64_t)B * Hq > (int64_t(1) << 30)) return ATTN_ERR_UNSUPPORTED;
  // the last query chunk visits every key/value chunk (causal or not)
  const int need = n_chunks > 1 ? n_chunks : 0;
  if (ws_slots < need) return ATTN_ERR_INVALID_ARG;
  if (need > 0 && (!ws_o || !ws_lse || !aligned(ws_o, 32) || !aligned(ws_lse, 4)))
    return ATTN_ERR_INVALID_ARG;
  const int64_t C = N / n_chunks;
  const uint64_t bh = (uint64_t)B * Hq, bhkv = (uint64_t)B * Hkv;
  const uint64_t slot_rows = bh * (uint64_t)C;
  std::vector<Span> dev = {span(q_d, bh * N * d * 2), span(k_d, bhkv * N * d * 2),
                           span(v_d, bhkv * N * d * 2), span(o_d, bh * N * d * 4),
                           span(lse_d, bh * N * 4)};
  if (need > 0) {
    dev.push_back(span(ws_o, need * slot_rows * d * 4));
    dev.push_back(span(ws_lse, need * slot_rows * 4));
  }
  for (size_t i = 0; i < dev.size(); ++i)
    for (size_t j = 0; j < i; ++j)
      if (overlap(dev[i], dev[j])) return ATTN_ERR_INVALID_ARG;
  attn_status_t inj = take_injected();
  if (inj != ATTN_OK) return inj;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaStream_t sh = h2d_stream ? static_cast<cudaStream_t>(h2d_stream) : s;
  cudaStream_t sd = d2h_stream ? static_cast<cudaStream_t>(d2h_stream) : s;
  const int P = n_chunks;

  // Arrival points of the copies in: each point is a group of chunks whose arrival is
  // marked by one event. Causal: Q_0, KV_0, Q_1, KV_1, ... - pair (i, kv < i) is ready
  // once Q_i is in, the diagonal pair (i, i) once KV_i is, so when the last chunk
  // arrives only one diagonal pair is left to compute. Non-causal (every query chunk
  // needs every key/value chunk): KV_0 .. KV_{P-1}, then Q_0, Q_1, ... - query chunk
  // i is ready once Q_i is in, and results leave while later Q chunks still arrive.
  const int n_points = 2 * P;
  auto q_point = [&](int i) { return causal ? 2 * i : P + i; };
  auto kv_point = [&](int c) { return causal ? 2 * c + 1 : c; };
  // events: [0] start, [1] end, [2 + t] arrival point t, [2 + n_points + i] result i final
  std::vector<cudaEvent_t> ev(2 + (size_t)n_points + P, nullptr);
  auto release = [&]() {
    for (cudaEvent_t e : ev)
      if (e) cudaEventDestroy(e);  // resources are released once pending work completes
  };
  for (auto& e : ev) {
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      e = nullptr;
      release();
      return ATTN_ERR_CUDA;
    }
  }
  attn_status_t st = ATTN_OK;
  auto cuda_ok = [&](cudaError_t e) {
    if (e != cudaSuccess && st == ATTN_OK) st = ATTN_ERR_CUDA;
    return st == ATTN_OK;
  };
  auto after = [&](cudaStream_t waiter, cudaEvent_t e, cudaStream_t signaller) {
    if (waiter == signaller) return true;  // stream order already covers it
    return cuda_ok(cudaEventRecord(e, signaller)) && cuda_ok(cudaStreamWaitEvent(waiter, e, 0));
  };
  // the copies in overwrite the staging buffers: after earlier work on `stream`
  // (the copies back wait for events recorded on `stream`, so they follow it anyway)
  after(sh, ev[0], s);

  // host -> device, one arrival point at a time: strided copies (B*H runs of C rows)
  const size_t pitch = (size_t)N * d * 2, width = (size_t)C * d * 2;
  auto copy_in = [&](void* dst, const void* src, int c, uint64_t runs) {
    const size_t off = (size_t)c * width;
    cuda_ok(cudaMemcpy2DAsync(static_cast<char*>(dst) + off, pitch,
                              static_cast<const char*>(src) + off, pitch, width, runs,
                              cudaMemcpyHostToDevice, sh));
  };
  for (int t = 0; t < n_points && st == ATTN_OK; ++t) {
    for (int c = 0; c < P; ++c) {
      if (kv_point(c) == t) {
        copy_in(k_d, k_h, c, bhkv);
        copy_in(v_d, v_h, c, bhkv);
      }
      if (q_point(c) == t) copy_in(q_d, q_h, c, bh);
    }
    if (st == ATTN_OK && sh != s) cuda_ok(cudaEventRecord(ev[2 + t], sh));
  }

  // Pairs launch at their arrival point (one batched launch per point); a query
  // chunk's partials go to partial slot j for its j-th key/value chunk in ring order
  // (chunk (i - j) mod P), are merged in that order once its last pair has run, and the
  // result goes back. A query chunk's pairs all run between two of its own points, and
  // chunks finish in order, so P partial slots serve every chunk.
  auto visits = [&](int i, int* kv_of_slot) {
    int nv = 0;
    for (int step = 0; step < P; ++step) {
      const int kv = ((i - step) % P + P) % P;
      if (causal && kv > i) continue;
      kv_of_slot[nv++] = kv;
    }
    return nv;
  };
  attn_pair_t pairs[ATTN_MAX_BATCH_PAIRS];
  const float* po[ATTN_MAX_BATCH_PAIRS];
  const float* pl[ATTN_MAX_BATCH_PAIRS];
  int kv_of_slot[ATTN_MAX_BATCH_PAIRS];
  for (int t = 0; t < n_points && st == ATTN_OK; ++t) {
    int np = 0;
    int finished = -1;  // the query chunk whose last pair runs at this point, if any
    for (int i = 0; i < P; ++i) {
      const int nv = visits(i, kv_of_slot);
      int last = -1;
      for (int j = 0; j < nv; ++j) {
        const int kv = kv_of_slot[j];
        const int ready = q_point(i) > kv_point(kv) ? q_point(i) : kv_point(kv);
        last = ready > last ? ready : last;
        if (ready != t) continue;
        float* o_j = nv == 1 ? o_d + (size_t)i * slot_rows * d : ws_o + (size_t)j * slot_rows * d;
        float* l_j = nv == 1 ? lse_d + (size_t)i * slot_rows : ws_lse + (size_t)j * slot_rows;
        pairs[np++] = attn_pair_t{i * C, C, kv * C, C, i * C, kv * C, o_j, l_j};
      }
      if (last == t) finished = i;
    }
    if (np == 0) continue;
    if (sh != s && !cuda_ok(cudaStreamWaitEvent(s, ev[2 + t], 0))) break;
    st = attn_fwd_partial_batch(q_d, k_d, v_d, B, Hq, Hkv, N, N, d, causal, scale, pairs, np, 0,
                                stream);
    if (st != ATTN_OK || finished < 0) continue;
    const int i = finished;
    float* o_i = o_d + (size_t)i * slot_rows * d;
    float* l_i = lse_d + (size_t)i * slot_rows;
    const int nv = visits(i, kv_of_slot);
    if (nv > 1) {
      for (int j = 0; j < nv; ++j) {
        po[j] = ws_o + (size_t)j * slot_rows * d;
        pl[j] = ws_lse + (size_t)j * slot_rows;
      }
      st = attn_merge(po, pl, nv, o_i, l_i, (int64_t)slot_rows, d, stream);
      if (st != ATTN_OK) break;
    }
    if (sd != s && !(cuda_ok(cudaEventRecord(ev[2 + n_points + i], s)) &&
                     cuda_ok(cudaStreamWaitEvent(sd, ev[2 + n_points + i], 0))))
      break;
    cuda_ok(cudaMemcpyAsync(o_h + (size_t)i * slot_rows * d, o_i, slot_rows * d * 4,
                            cudaMemcpyDeviceToHost, sd));
    cuda_ok(cudaMemcpyAsync(lse_h + (size_t)i * slot_rows, l_i, slot_rows * 4,
                            cudaMemcpyDeviceToHost, sd));
  }
  // later work on `stream` waits for the last copy back
  if (st == ATTN_OK) after(s, ev[1], sd);
  release();
  return st;
}

attn_status_t attn_debug_exp2(const float* x, float* y, int64_t n, int use_poly, void* stream) {
  if (!x || !y || n < 1 || (use_poly != 0 && use_poly != 1)) return ATTN_ERR_INVALID_ARG;
  if (!aligned(x, 4) || !aligned(y, 4)) return ATTN_ERR_INVALID_ARG;
  if (overlap(span(x, (uint64_t)n * 4), span(y, (uint64_t)n * 4))) return ATTN_ERR_INVALID_ARG;
  return static_cast<attn_status_t>(
      osx::launch_exp2_probe(x, y, n, use_poly, static_cast<cudaStream_t>(stream)));
}

uint64_t attn_launch_count(void) { return osx::launch_count(); }

}  // extern "C"
