// attn_internal.h - interface between the C ABI layer (attn_api.cu) and the kernel
// translation unit (attn_kernels.cu). Not installed; not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

namespace osx {

// One (query chunk, key/value chunk) pair of a launch; rows are tensor-map rows.
struct PairLaunch {
  long long q_start, q_len, kv_start, kv_len, q_off, kv_off;
  float* o;
  float* lse;
};

// One attention launch over up to kMaxPairs pairs sharing the q/k/v tensor maps;
// arguments have already been validated by the ABI layer. The maps span q_rows
// (resp. kv_rows) rows of [B*H][rows][d] views with row strides q_ld / kv_ld.
struct FwdLaunch {
  const void* q;
  const void* k;
  const void* v;
  int B, Hq, Hkv;
  long long q_rows, kv_rows, q_ld, kv_ld;
  int d;
  int causal;
  float scale;
  int accumulate;  // o/lse are in/out accumulators (see attn_fwd_partial_acc)
  int n_pairs;
  const PairLaunch* pairs;
};

// Returns 0 (ATTN_OK) or an attn_status_t failure code.
int launch_fwd(const FwdLaunch& a, cudaStream_t stream);
int launch_merge(const float* const* o_parts, const float* const* lse_parts, int n_parts,
                 float* o, float* lse, long long rows, int d, cudaStream_t stream);
// Launches the failure-path check kernel (a bounded wait that must run out).
int launch_wait_probe(long long limit_cycles, cudaStream_t stream);
// Launches the exponential check kernel (y = 2^x by the polynomial or by ex2.approx).
int launch_exp2_probe(const float* x, float* y, long long n, int use_poly, cudaStream_t stream);
// Reads (and optionally clears) the device status word of the current device.
int read_device_status(unsigned* out, int reset);
uint64_t launch_count();

}  // namespace osx
