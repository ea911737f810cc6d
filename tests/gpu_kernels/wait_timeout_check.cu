// Test harness (not part of the library): drives the bounded mbarrier wait
// every kernel of the library uses (ptx.cuh, mbar_wait) into each of its
// exits on the GPU -- the time limit, another thread's abort flag, and a
// normal arrival -- and reports what the waits returned, how long they took
// and the error word they left.  Every wait and spin here is bounded by the
// global timer; nothing faults, traps or hangs.
#include <cstdint>
#include <cuda_runtime.h>
#include "ptx.cuh"

namespace {

struct WaitResult {
  int ok_timeout, ok_abort, ok_arrived, first_code;
  unsigned long long ns_timeout, ns_abort, ns_arrived;
};

// spin on the global timer for ns (bounded by construction)
__device__ void sleep_ns(unsigned long long ns) {
  const uint64_t t0 = swa::globaltimer();
  while (swa::globaltimer() - t0 < ns) {
  }
}

// warp 0 lane 0 waits; warp 1 lane 0 raises the abort flag / arrives on cue
__global__ void wait_exits_kernel(WaitResult* out, unsigned long long limit_ns, unsigned long long delay_ns) {
  __shared__ uint64_t never, later;
  __shared__ int abort_flag, cue;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    swa::mbar_init(&never, 1);  // nothing ever arrives on it
    swa::mbar_init(&later, 1);  // warp 1 arrives once, after a delay
    abort_flag = 0;
    cue = 0;
    swa::fence_mbar_init();
  }
  __syncthreads();
  volatile int* af = &abort_flag;
  volatile int* vcue = &cue;
  if (warp == 0 && lane == 0) {
    // 1. the time limit: no arrival, no abort
    uint64_t t0 = swa::globaltimer();
    bool ok = swa::mbar_wait(&never, 0, af, limit_ns);
    out->ns_timeout = swa::globaltimer() - t0;
    out->ok_timeout = ok;
    if (!ok) swa::record_error(9901);
    swa::record_error(9902);  // the first recorded code stays
    // 2. another thread's abort flag ends a wait long before its limit
    *vcue = 1;
    t0 = swa::globaltimer();
    ok = swa::mbar_wait(&never, 0, af, 20 * limit_ns);
    out->ns_abort = swa::globaltimer() - t0;
    out->ok_abort = ok;
    // 3. a normal arrival completes the wait
    *af = 0;
    *vcue = 2;
    t0 = swa::globaltimer();
    ok = swa::mbar_wait(&later, 0, af, 20 * limit_ns);
    out->ns_arrived = swa::globaltimer() - t0;
    out->ok_arrived = ok;
  } else if (warp == 1 && lane == 0) {
    const uint64_t t0 = swa::globaltimer();
    const uint64_t give_up = 40 * limit_ns;  // bounds both cue spins
    while (*vcue < 1 && swa::globaltimer() - t0 < give_up) {
    }
    sleep_ns(delay_ns);
    *af = 1;
    while (*vcue < 2 && swa::globaltimer() - t0 < give_up) {
    }
    sleep_ns(delay_ns);
    swa::mbar_arrive(&later);
  }
  __syncthreads();
  if (threadIdx.x == 0) out->first_code = swa::g_device_error;
}

}  // namespace

extern "C" __attribute__((visibility("default"))) int wait_exits_run(void* result, unsigned long long limit_ns,
                                                                  unsigned long long delay_ns) {
  WaitResult* d = nullptr;
  cudaError_t e = cudaMalloc(&d, sizeof(WaitResult));
  if (e != cudaSuccess) return (int)e;
  const int zero = 0;
  e = cudaMemcpyToSymbol(swa::g_device_error, &zero, sizeof(int));
  if (e == cudaSuccess) {
    wait_exits_kernel<<<1, 64>>>(d, limit_ns, delay_ns);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(result, d, sizeof(WaitResult), cudaMemcpyDeviceToHost);
  cudaFree(d);
  return (int)e;
}

extern "C" __attribute__((visibility("default"))) int wait_error_word(void) {
  int v = -1;
  if (cudaMemcpyFromSymbol(&v, swa::g_device_error, sizeof(int)) != cudaSuccess) return -1;
  return v;
}
