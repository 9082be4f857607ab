// Measurement support: the effective SM clock during a timed region; and a
// self-test of the bounded waits' failure path.
//
// One thread records (%globaltimer, %clock64) pairs about every period_ns
// for duration_ns, sleeping in between (the warp issues almost nothing and
// uses no shared memory, so it shares its SM with the kernels being timed).
// Cycles over nanoseconds between two records is the clock of that SM over
// the interval.  Every wait is bounded: a record is taken after at most
// kMaxSleeps sleeps even if the timer has not reached its target.
#include <cstdint>
#include <cuda_runtime.h>

#include "bench_probe.h"
#include "sm100.cuh"

namespace ptpc {

namespace {

constexpr int kMaxSleeps = 4096;   // per record: at most ~80 ms of 20 us sleeps
constexpr unsigned kSleepNs = 20000;

__global__ void clock_probe_kernel(unsigned long long *__restrict__ out, int max_records, uint64_t period_ns,
                                   uint64_t duration_ns, int *__restrict__ count) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const uint64_t t0 = global_timer_ns();
  int n = 0;
  while (n < max_records) {
    out[2 * n] = global_timer_ns();
    out[2 * n + 1] = clock64();
    const uint64_t t = out[2 * n];
    ++n;
    if (t - t0 >= duration_ns) break;
    const uint64_t target = t0 + (uint64_t)n * period_ns;
    for (int i = 0; i < kMaxSleeps && global_timer_ns() < target; ++i) __nanosleep(kSleepNs);
  }
  *count = n;
}

// Status bit set by the wait self-test below.
constexpr uint32_t kStatusTimeoutSelftest = 1u << 3;

// One thread waits, with the kernels' own bounded mbar_wait, on a barrier
// that nothing ever arrives at: the wait runs out after its limit (2 s of
// %globaltimer), the kernel records the timeout in the status word and
// returns.  Nothing faults or hangs; the context stays usable.
__global__ void wait_timeout_selftest_kernel(uint32_t *status) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_barrier_init();
  if (!mbar_wait(&bar, 0)) atomicOr(status, kStatusTimeoutSelftest);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(uint32_t *status, cudaStream_t st) {
  wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(status);
  return cudaGetLastError();
}

cudaError_t launch_clock_probe(unsigned long long *out, int max_records, uint64_t period_ns, uint64_t duration_ns,
                               int *count, cudaStream_t st) {
  // Keep the probe's SM configured for the largest shared memory: a GEMM CTA
  // (about 210 KB) must still fit beside it.
  cudaError_t e = cudaFuncSetAttribute(clock_probe_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                       (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  clock_probe_kernel<<<1, 32, 0, st>>>(out, max_records, period_ns, duration_ns, count);
  return cudaGetLastError();
}

}  // namespace ptpc
