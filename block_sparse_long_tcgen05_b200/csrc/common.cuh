// Shared definitions of the MSA CUDA library: status codes, the device error word,
// and fixed limits.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/msa.h"

namespace msa {

// Longest time any single wait on an mbarrier may take before the kernel gives up,
// records MSA_ERR_TIMEOUT and returns (every pipeline step of these kernels completes
// in microseconds; two seconds is a hang).
constexpr uint64_t kWaitLimitNs = 2000000000ull;
// Longest time a warp sleeps in one mbarrier try_wait before it re-checks the time and the
// abort flag.
constexpr uint64_t kSuspendHintNs = 1000000ull;

// Time limit of the waits that gate new work, read by every pipelined kernel when it starts
// (msa_set_wait_limit_ns changes it; drains always use kWaitLimitNs).
__device__ uint64_t g_msa_wait_limit_ns = kWaitLimitNs;

// Kernel ids recorded in the device error word (bits 8..15).
enum KernelId : int {
  kKidIndexScore = 1,
  kKidTopk = 2,
  kKidCsr = 3,
  kKidKvOuter = 4,
  kKidMerge = 5,
  kKidDecodeScan = 6,
  kKidDecodeAttn = 7,
  kKidKl = 8,
};

// Device error word: low byte = first msa_status_t recorded, next byte = kernel id.
// Lives in the library's own static device memory, one per device. (The library is a
// single translation unit, msa_api.cu, which includes every kernel header.)
__device__ unsigned int g_msa_error = 0u;

__device__ __forceinline__ void record_error(int status, int kernel_id) {
  atomicCAS(&g_msa_error, 0u, static_cast<unsigned int>(status & 0xFF) | (static_cast<unsigned int>(kernel_id & 0xFF) << 8));
}

}  // namespace msa
