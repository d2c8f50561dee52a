// attn_internal.h - interface between the C ABI layer (attn_api.cu) and the kernel
// translation unit (attn_kernels.cu). Not installed; not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

namespace osx {

// One attention launch over a (query chunk, key/value chunk) pair; arguments have
// already been validated by the ABI layer.
struct FwdLaunch {
  const void* q;
  const void* k;
  const void* v;
  float* o;
  float* lse;
  int B, Hq, Hkv;
  long long Nq, Nkv, q_ld, kv_ld, q_off, kv_off;
  int d;
  int causal;
  float scale;
  int accumulate;  // o/lse are an in/out accumulator (see attn_fwd_partial_acc)
};

// Returns 0 (ATTN_OK) or an attn_status_t failure code.
int launch_fwd(const FwdLaunch& a, cudaStream_t stream);
int launch_merge(const float* const* o_parts, const float* const* lse_parts, int n_parts,
                 float* o, float* lse, long long rows, int d, cudaStream_t stream);
// Launches the failure-path check kernel (a bounded wait that must run out).
int launch_wait_probe(long long limit_cycles, cudaStream_t stream);
// Reads (and optionally clears) the device status word of the current device.
int read_device_status(unsigned* out, int reset);
uint64_t launch_count();

}  // namespace osx
