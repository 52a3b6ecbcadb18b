// Shared device state and small helpers for the sbsa kernels.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace sbsa {

// Device error word, one per device (module-scope __device__ variable).  Bits are the
// sbsa_status codes (1 << code).  Read and cleared by sbsa_check().
__device__ unsigned int g_error_bits;

// When a bounded wait in one CTA expires, it stores its launch's epoch here so that
// every other CTA of the same launch gives up at once instead of waiting out its own
// limit.  Launches carry distinct epochs, so an old abort never affects a new launch.
__device__ unsigned int g_abort_epoch;

// Result flag of the CSR validation kernel (sbsa_validate_csr is synchronous, so
// concurrent validations on one device must not overlap).
__device__ unsigned int g_csr_bad;

constexpr unsigned int kErrTimeout = 1u << 5;   // SBSA_ERR_TIMEOUT
constexpr unsigned int kErrBadIndex = 1u << 6;  // SBSA_ERR_BAD_INDEX

// Upper bound on any single wait inside a kernel.  Every legitimate wait is
// microseconds long; this only ends a kernel whose pipeline has stalled.  The waits a
// CTA makes after giving up, for its own copies and tensor-core work still in flight
// (the drain), always use this limit.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s

// Limit of the pipeline waits (everything but the drain) of the attention, selection,
// RoPE + pooling and FP8 quantizer kernels, per device; kWaitLimitNs unless
// sbsa_set_pipeline_wait_ns changed it.  0 makes a pipeline wait give up unless its
// barrier has already completed at the first test, which lets a test drive the
// give-up path without a stalled pipeline.
__device__ unsigned long long g_pipe_wait_ns = kWaitLimitNs;

__device__ __forceinline__ uint64_t pipe_wait_ns() {
    return *reinterpret_cast<volatile unsigned long long*>(&g_pipe_wait_ns);
}

__device__ __forceinline__ void raise_error(unsigned int bits) { atomicOr(&g_error_bits, bits); }

__device__ __forceinline__ bool launch_aborted(unsigned int epoch) {
    return *reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch;
}

__device__ __forceinline__ void abort_launch(unsigned int epoch) {
    raise_error(kErrTimeout);
    atomicExch(&g_abort_epoch, epoch);
}

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

}  // namespace sbsa
