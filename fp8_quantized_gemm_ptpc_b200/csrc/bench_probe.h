// Measurement and self-test support (bench_probe.cu), kept apart from the kernels' interface.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace ptpc {

// (globaltimer ns, SM clock cycles) pairs about every period_ns for
// duration_ns into out[2 * max_records]; the number written goes to *count.
cudaError_t launch_clock_probe(unsigned long long *out, int max_records, uint64_t period_ns, uint64_t duration_ns,
                               int *count, cudaStream_t st);

// Launches a kernel whose bounded wait must run out (about 2 s) and record a
// timeout bit in *status.
cudaError_t launch_wait_timeout_selftest(uint32_t *status, cudaStream_t st);

}  // namespace ptpc
