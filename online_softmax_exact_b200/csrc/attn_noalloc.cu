// attn_noalloc.cu - attn_ring_fwd_host_noalloc: the host-buffer ring call for callers
// that cannot allocate device memory.
//
// attn_ring_fwd_host needs device memory besides its host inputs and outputs: staging
// buffers for Q, K, V and the result, and one partial-result slot per chunk. Here all
// of it lives in one fixed array of this library's own device data (below), so the
// call allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
// Callers that need this are, for example, code running in a process whose device
// memory is owned by another allocator (a framework's caching allocator holding the
// free memory, or a fixed memory budget per component), and code on a latency-critical
// path where cudaMalloc/cudaFree would synchronise the device.
//
// The array is sized once, at build time, to ATTN_NOALLOC_SCRATCH_BYTES; every GPU on
// which the library is loaded holds it until the process exits. Calls share it, so
// calls whose work overlaps on the GPU race (see attn.h).
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/attn.h"

namespace {

constexpr uint64_t kScratchBytes = ATTN_NOALLOC_SCRATCH_BYTES;

// The scratch array. In host code its name stands for a host-side shadow, not a device
// address: the device address comes from cudaGetSymbolAddress (scratch_base below).
__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_base[kMaxDevices];  // device address of the array, per device, once known
std::mutex g_scratch_mutex;

// Per-device set-up, on the first call with that device current: look up the device
// address of the scratch array.
attn_status_t scratch_base(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_base[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return ATTN_ERR_CUDA;
    g_scratch_base[dev] = p;
  }
  *out = g_scratch_base[dev];
  return ATTN_OK;
}

uint64_t round256(uint64_t x) { return (x + 255u) & ~uint64_t(255); }

}  // namespace

extern "C" attn_status_t attn_ring_fwd_host_noalloc(const void* q_h, const void* k_h,
                                                    const void* v_h, float* o_h, float* lse_h,
                                                    int B, int Hq, int Hkv, int64_t N, int d,
                                                    int n_chunks, int causal, float scale,
                                                    void* stream, void* h2d_stream,
                                                    void* d2h_stream) {
  // the checks attn_ring_fwd_host makes on these arguments, made here first so that a
  // bad call neither touches the device nor is mistaken for a size the array lacks
  if (!q_h || !k_h || !v_h || !o_h || !lse_h) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || N < 1) return ATTN_ERR_INVALID_ARG;
  if (n_chunks < 1 || N % n_chunks != 0) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (n_chunks > ATTN_MAX_BATCH_PAIRS) return ATTN_ERR_UNSUPPORTED;

  // device memory the call needs, carved from the array in 256-byte aligned pieces
  const uint64_t bh = (uint64_t)B * (uint64_t)Hq, bhkv = (uint64_t)B * (uint64_t)Hkv;
  if (bh > kScratchBytes || (uint64_t)N > kScratchBytes || bh * (uint64_t)N > kScratchBytes)
    return ATTN_ERR_UNSUPPORTED;
  const uint64_t rows_q = bh * (uint64_t)N, rows_kv = bhkv * (uint64_t)N;
  const int slots = n_chunks > 1 ? n_chunks : 0;
  const uint64_t slot_rows = rows_q / (uint64_t)n_chunks;
  uint64_t off = 0;
  const uint64_t off_q = off;
  off += round256(rows_q * d * 2);
  const uint64_t off_k = off;
  off += round256(rows_kv * d * 2);
  const uint64_t off_v = off;
  off += round256(rows_kv * d * 2);
  const uint64_t off_o = off;
  off += round256(rows_q * d * 4);
  const uint64_t off_lse = off;
  off += round256(rows_q * 4);
  const uint64_t off_wo = off;
  off += round256((uint64_t)slots * slot_rows * d * 4);
  const uint64_t off_wl = off;
  off += round256((uint64_t)slots * slot_rows * 4);
  if (off > kScratchBytes) return ATTN_ERR_UNSUPPORTED;

  void* base = nullptr;
  attn_status_t st = scratch_base(&base);
  if (st != ATTN_OK) return st;
  unsigned char* s = static_cast<unsigned char*>(base);
  // nothing in the array needs clearing: the call writes every byte it reads first (the
  // copies fill the staging rows, the partials their slots, the merges the result);
  // bytes beyond a chunk that the kernels load are never used (see attn.h)
  return attn_ring_fwd_host(q_h, k_h, v_h, o_h, lse_h, s + off_q, s + off_k, s + off_v,
                            reinterpret_cast<float*>(s + off_o),
                            reinterpret_cast<float*>(s + off_lse),
                            slots ? reinterpret_cast<float*>(s + off_wo) : nullptr,
                            slots ? reinterpret_cast<float*>(s + off_wl) : nullptr, slots, B, Hq,
                            Hkv, N, d, n_chunks, causal, scale, stream, h2d_stream, d2h_stream);
}
