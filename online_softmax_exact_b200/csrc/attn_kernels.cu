// attn_kernels.cu - the library's only device translation unit: kernel instantiations,
// per-device set-up, and launchers.
#include <atomic>
#include <cmath>
#include <mutex>

#include "../../include/attn.h"
#include "attn_fwd_kernel.cuh"
#include "attn_internal.h"
#include "attn_merge_kernel.cuh"
#include "tma_host.h"

namespace osx {

// Device status word (one per device that loads the library): bounded waits that run
// out record kDevTimeout here. Read through read_device_status().
__device__ unsigned g_device_status;

// Failure-path check: one thread waits on an mbarrier that nothing arrives on, through
// the same bounded wait the attention kernel uses, with a short limit. The wait runs
// out, records kDevTimeout in the status word and the kernel returns.
__global__ void wait_probe_kernel(unsigned* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar_storage;
  __shared__ int abort_storage;
  if (threadIdx.x == 0) {
    abort_storage = 0;
    mbar_init(smem_u32(&bar_storage), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    mbar_wait_limit(smem_u32(&bar_storage), 0, &abort_storage, status, limit_ns);
  __syncthreads();
}

// Check of the exponentials the softmax uses: y = 2^x through the FMA-pipe polynomial
// (use_poly != 0, two values per call as in the kernel) or through ex2.approx.
__global__ void exp2_probe_kernel(const float* __restrict__ x, float* __restrict__ y,
                                  long long n, int use_poly) {
  const long long stride = 2ll * gridDim.x * blockDim.x;
  for (long long i = 2ll * (blockIdx.x * (long long)blockDim.x + threadIdx.x); i < n; i += stride) {
    const bool two = i + 1 < n;
    const float x0 = x[i], x1 = two ? x[i + 1] : 0.f;
    float y0, y1;
    if (use_poly) {
      f2_unpack(exp2_poly_f32x2(f2_pack(x0, x1)), y0, y1);
    } else {
      y0 = ex2_approx(x0);
      y1 = ex2_approx(x1);
    }
    y[i] = y0;
    if (two) y[i + 1] = y1;
  }
}

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  int clock_khz = 0;           // peak SM clock
  long long l2_bytes = 0;      // L2 cache size
  unsigned* status = nullptr;  // device address of g_device_status
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;
std::atomic<uint64_t> g_launches{0};

// Per-device set-up, once per device with that device current: SM count, the device
// address of the status word, and the dynamic shared-memory opt-in of each kernel.
int device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  DeviceInfo& di = g_dev[dev];
  if (!di.ready) {
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!di.ready) {
      int sms = 0, khz = 0, l2 = 0;
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return ATTN_ERR_CUDA;
      if (cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess || l2 <= 0)
        l2 = 126 << 20;
      if (cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev) != cudaSuccess || khz <= 0)
        khz = 2000000;
      void* st = nullptr;
      if (cudaGetSymbolAddress(&st, g_device_status) != cudaSuccess) return ATTN_ERR_CUDA;
      if (cudaFuncSetAttribute(attn_fwd_kernel<64>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)FwdCfg<64>::kSmemBytes) != cudaSuccess)
        return ATTN_ERR_CUDA;
      if (cudaFuncSetAttribute(attn_fwd_kernel<128>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)FwdCfg<128>::kSmemBytes) != cudaSuccess)
        return ATTN_ERR_CUDA;
      di.num_sms = sms;
      di.clock_khz = khz;
      di.l2_bytes = l2;
      di.status = static_cast<unsigned*>(st);
      di.ready = true;
    }
  }
  *out = &di;
  return ATTN_OK;
}

// three tensor maps plus the parameter block stay within the classic 4 KB of kernel
// parameters
static_assert(3 * sizeof(CUtensorMap) + sizeof(FwdParams) <= 4096, "kernel parameters");

// Key tiles that one (batch, head) of a pair visits over all its 256-row blocks, and the
// most that one block visits.
double pair_tiles(const PairLaunch& s, int causal) {
  const long long tiles = (s.kv_len + 127) / 128;
  const long long nqp = (s.q_len + 255) / 256;
  if (!causal) return (double)tiles * nqp;
  double sum = 0.0;
  for (long long qp = 0; qp < nqp; ++qp) {
    long long last = qp * 256 + 255;
    if (last > s.q_len - 1) last = s.q_len - 1;
    const long long lim = s.q_off + last - s.kv_off;
    if (lim < 0) continue;
    const long long n = lim / 128 + 1;
    sum += (double)(n < tiles ? n : tiles);
  }
  return sum;
}

long long heaviest_unit_tiles(const PairLaunch& s, int causal) {
  const long long tiles = (s.kv_len + 127) / 128;
  if (!causal) return tiles;
  const long long lim = s.q_off + s.q_len - 1 - s.kv_off;
  if (lim < 0) return 0;
  const long long n = lim / 128 + 1;
  return n < tiles ? n : tiles;
}

template <int D>
int launch_fwd_d(const FwdLaunch& a, const DeviceInfo& di, cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  if (!encode_rows_bf16(&tq, a.q, (uint64_t)a.B * a.Hq, a.q_rows, a.q_ld, D, 128) ||
      !encode_rows_bf16(&tk, a.k, (uint64_t)a.B * a.Hkv, a.kv_rows, a.kv_ld, D, 128) ||
      !encode_rows_bf16(&tv, a.v, (uint64_t)a.B * a.Hkv, a.kv_rows, a.kv_ld, D, 128))
    return ATTN_ERR_UNSUPPORTED;
  if (a.n_pairs < 1 || a.n_pairs > kMaxPairs) return ATTN_ERR_UNSUPPORTED;
  FwdParams p;
  p.status = di.status;
  p.BH = a.B * a.Hq;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.group = a.Hq / a.Hkv;
  p.causal = a.causal;
  p.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634);
  p.accumulate = a.accumulate;
  p.kv_rows = static_cast<int>(a.kv_rows);
  p.n_pairs = a.n_pairs;
  p.o_vec8 = 1;
  long long units = 0;
  for (int i = 0; i < kMaxPairs; ++i) {
    PairDesc& d = p.pair[i];
    if (i >= a.n_pairs) {
      d = PairDesc{};
      p.unit_end[i] = static_cast<int>(units);
      continue;
    }
    const PairLaunch& s = a.pairs[i];
    d.o = s.o;
    d.lse = s.lse;
    d.q_off = s.q_off;
    d.kv_off = s.kv_off;
    d.q_row0 = static_cast<int>(s.q_start);
    d.kv_row0 = static_cast<int>(s.kv_start);
    d.Nq = static_cast<int>(s.q_len);
    d.Nkv = static_cast<int>(s.kv_len);
    {
      // uniform: even the first row block sees every key tile
      const long long tiles = (s.kv_len + 127) / 128;
      const long long last_row0 = (s.q_len < 256 ? s.q_len : 256) - 1;
      const long long lim0 = s.q_off + last_row0 - s.kv_off;
      d.uniform = (!a.causal || lim0 >= (tiles - 1) * 128) ? 1 : 0;
    }
    // a uniform pair joins the previous pair's group if that one is uniform too and
    // reads the same key/value rows with the same shapes
    d.group_first = i;
    d.group_n = 1;
    if (i > 0 && d.uniform && p.pair[i - 1].uniform && p.pair[i - 1].kv_row0 == d.kv_row0 &&
        p.pair[i - 1].Nkv == d.Nkv && p.pair[i - 1].Nq == d.Nq) {
      d.group_first = p.pair[i - 1].group_first;
      d.group_n = i - d.group_first + 1;
      for (int g = d.group_first; g < i; ++g) p.pair[g].group_n = d.group_n;
    }
    if ((reinterpret_cast<uintptr_t>(s.o) % 32) != 0) p.o_vec8 = 0;
    units += ((s.q_len + 255) / 256) * (long long)p.BH;
    if (units > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    p.unit_end[i] = static_cast<int>(units);
  }
  const int grid = units < di.num_sms ? static_cast<int>(units) : di.num_sms;
  using Cfg = FwdCfg<D>;
  attn_fwd_kernel<D><<<grid, Cfg::kThreads, Cfg::kSmemBytes, stream>>>(tq, tk, tv, p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return ATTN_OK;
}

template <int D, int G>
int launch_merge_dg(const MergeParams& p, const DeviceInfo& di, cudaStream_t stream) {
  constexpr int rows_per_block = (256 / (D / 8)) * (8 / G);
  long long blocks = (p.rows + rows_per_block - 1) / rows_per_block;
  const long long cap = (long long)di.num_sms * 4;
  if (blocks > cap) blocks = cap;
  attn_merge_kernel<D, G><<<(unsigned)blocks, 256, 0, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return ATTN_OK;
}

template <int D>
int launch_merge_d(const MergeParams& p, const DeviceInfo& di, cudaStream_t stream) {
  if (p.n <= 2) return launch_merge_dg<D, 2>(p, di, stream);
  if (p.n <= 4) return launch_merge_dg<D, 4>(p, di, stream);
  return launch_merge_dg<D, 8>(p, di, stream);
}

}  // namespace

namespace {

int launch_fwd_one(const FwdLaunch& a, const DeviceInfo& di, cudaStream_t stream) {
  switch (a.d) {
    case 64: return launch_fwd_d<64>(a, di, stream);
    case 128: return launch_fwd_d<128>(a, di, stream);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

// Key/value heads per launch for a one-pair call with a causal cut whose K/V (all heads)
// exceed three quarters of L2: the fewest whose K/V fit in three quarters of L2 while the
// launch's heaviest work unit stays within a CTA's share of it (each launch runs its units
// heaviest first, so its heaviest start at once); 0: one launch.
// The kernel runs a pair's units row block by row block, heaviest first, all heads side by
// side; once the CTAs drift apart they stream different heads' K/V at different key
// positions, and K/V that do not fit in L2 are then read from DRAM many times over
// (measured on B200: 203 GB of reads for 0.54 GB of K/V in the 128k GQA call, 17 GB for
// 0.5 GB in a 32k causal call of 32 heads). Launching a few key/value heads at a time
// keeps the K/V being read within L2: +8% and +6.5% on those two calls.
int kv_heads_per_launch(const FwdLaunch& a, const DeviceInfo& di) {
  if (a.n_pairs != 1 || !a.causal) return 0;
  const PairLaunch& s = a.pairs[0];
  const double kv_head_bytes = (double)s.kv_len * a.d * 4.0;  // K and V of one head
  const double budget = 0.75 * (double)di.l2_bytes;
  if (kv_head_bytes * a.B * a.Hkv <= budget) return 0;
  {
    // no causal cut inside the pair (even its first row block sees every key tile): the
    // kernel runs such pairs head by head already
    const long long kv_tiles = (s.kv_len + 127) / 128;
    const long long last_row0 = (s.q_len < 256 ? s.q_len : 256) - 1;
    if (s.q_off + last_row0 - s.kv_off >= (kv_tiles - 1) * 128) return 0;
  }
  const double tiles = pair_tiles(s, a.causal);  // one head's key tiles over all units
  const double heaviest = (double)heaviest_unit_tiles(s, a.causal);
  const int group = a.Hq / a.Hkv;
  const long long qp = (s.q_len + 255) / 256;
  for (int k = 1; k < a.Hkv; ++k) {
    if (a.Hkv % k != 0) continue;
    if (k * kv_head_bytes > budget) break;
    const long long units = qp * k * group;
    const double ctas = (double)(units < di.num_sms ? units : di.num_sms);
    if (heaviest <= tiles * k * group / ctas) return k;
  }
  return 0;
}

}  // namespace

int launch_fwd(const FwdLaunch& a, cudaStream_t stream) {
  DeviceInfo* di = nullptr;
  int rc = device_info(&di);
  if (rc != ATTN_OK) return rc;
  const int k = kv_heads_per_launch(a, *di);
  if (k == 0) return launch_fwd_one(a, *di, stream);
  // the same pair over bands of k key/value heads (and their query heads), one launch
  // each: every band's rows of Q, K, V, O and LSE are contiguous
  const int group = a.Hq / a.Hkv;
  const PairLaunch& s = a.pairs[0];
  for (int b = 0; b < a.B; ++b) {
    for (int g = 0; g < a.Hkv; g += k) {
      const long long qh = (long long)b * a.Hq + (long long)g * group;  // first query head
      const long long kvh = (long long)b * a.Hkv + g;                  // first K/V head
      PairLaunch pr = s;
      pr.o = s.o + qh * s.q_len * a.d;
      pr.lse = s.lse + qh * s.q_len;
      FwdLaunch band = a;
      band.q = static_cast<const char*>(a.q) + qh * a.q_ld * a.d * 2;
      band.k = static_cast<const char*>(a.k) + kvh * a.kv_ld * a.d * 2;
      band.v = static_cast<const char*>(a.v) + kvh * a.kv_ld * a.d * 2;
      band.B = 1;
      band.Hq = k * group;
      band.Hkv = k;
      band.pairs = &pr;
      rc = launch_fwd_one(band, *di, stream);
      if (rc != ATTN_OK) return rc;
    }
  }
  return ATTN_OK;
}

int launch_merge(const float* const* o_parts, const float* const* lse_parts, int n_parts,
                 float* o, float* lse, long long rows, int d, cudaStream_t stream) {
  DeviceInfo* di = nullptr;
  int rc = device_info(&di);
  if (rc != ATTN_OK) return rc;
  MergeParams p;
  for (int i = 0; i < kMaxMergeParts; ++i) {
    p.o[i] = i < n_parts ? o_parts[i] : nullptr;
    p.lse[i] = i < n_parts ? lse_parts[i] : nullptr;
  }
  p.out_o = o;
  p.out_lse = lse;
  p.rows = rows;
  p.n = n_parts;
  switch (d) {
    case 64: return launch_merge_d<64>(p, *di, stream);
    case 128: return launch_merge_d<128>(p, *di, stream);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

int launch_wait_probe(long long limit_cycles, cudaStream_t stream) {
  DeviceInfo* di = nullptr;
  int rc = device_info(&di);
  if (rc != ATTN_OK) return rc;
  // the device's wait limit is in nanoseconds: convert at the peak SM clock
  const unsigned long long ns =
      static_cast<unsigned long long>(limit_cycles) * 1000000ull / (unsigned)di->clock_khz + 1;
  wait_probe_kernel<<<1, 32, 0, stream>>>(di->status, ns);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return ATTN_OK;
}

int launch_exp2_probe(const float* x, float* y, long long n, int use_poly, cudaStream_t stream) {
  DeviceInfo* di = nullptr;
  int rc = device_info(&di);
  if (rc != ATTN_OK) return rc;
  long long blocks = (n + 511) / 512;
  if (blocks > (long long)di->num_sms * 8) blocks = (long long)di->num_sms * 8;
  exp2_probe_kernel<<<(unsigned)blocks, 256, 0, stream>>>(x, y, n, use_poly);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return ATTN_OK;
}

int read_device_status(unsigned* out, int reset) {
  if (cudaMemcpyFromSymbol(out, g_device_status, sizeof(unsigned)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (reset) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(unsigned)) != cudaSuccess)
      return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

uint64_t launch_count() { return g_launches.load(std::memory_order_relaxed); }

}  // namespace osx
