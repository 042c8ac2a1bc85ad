// Test-only probe of the library's time-bounded waits (pa_wait.cuh), the ones
// the prefill and decode kernels use: it makes them run out on purpose, with
// a short limit, on a barrier and a flag that nothing will ever complete, and
// reports what each wait returned.  Nothing here can hang: every wait has a
// limit of at most `other_ns`.
#include <cuda_runtime.h>

#include "pa_wait.cuh"

// One CTA of two warps sharing an mbarrier (expected arrivals: 1) and a flag.
//   mode 0: warp 0 waits on the barrier with limit `limit_ns`; nothing
//           arrives.  Warp 1 spins on the flag, which nothing sets, with the
//           longer limit `other_ns`: it must give up early, when warp 0 raises
//           the CTA's abort flag.
//   mode 1: the same with the roles swapped: warp 1's flag spin runs out
//           first and warp 0's barrier wait gives up on the abort flag.
//   mode 2: control: warp 1 arrives on the barrier after a short sleep and
//           sets the flag; both waits succeed and no status bit is set.
// result[0] = barrier wait's return value, result[1] = flag spin's return
// value, result[2] = the abort flag at the end, result[3] = warp 0's wait time
// in microseconds, result[4] = warp 1's.
__global__ void wait_timeout_probe_kernel(int* status, int* result, unsigned long long limit_ns,
                                          unsigned long long other_ns, int mode) {
  __shared__ __align__(8) unsigned long long bar;
  __shared__ int flag, abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t b = (uint32_t)__cvta_generic_to_shared(&bar);
  if (threadIdx.x == 0) {
    pa::mbar_init(b, 1);
    flag = 0;
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  volatile int* vabort = &abort_flag;
  volatile int* vflag = &flag;
  if (warp == 0) {
    const unsigned long long lim = mode == 0 ? limit_ns : other_ns;
    const uint64_t t0 = pa::globaltimer();
    const bool ok = pa::wait_bar(b, 0, vabort, status, lim);
    const uint64_t t1 = pa::globaltimer();
    if (lane == 0) {
      result[0] = ok ? 1 : 0;
      result[3] = (int)((t1 - t0) / 1000);
    }
  } else {
    if (mode == 2 && lane == 0) {
      __nanosleep(100000);
      *vflag = 1;
      pa::mbar_arrive(b);
    }
    __syncwarp();
    const unsigned long long lim = mode == 1 ? limit_ns : other_ns;
    const uint64_t t0 = pa::globaltimer();
    const bool ok = pa::spin_until([&] { return *vflag != 0; }, vabort, status, lim);
    const uint64_t t1 = pa::globaltimer();
    if (lane == 0) {
      result[1] = ok ? 1 : 0;
      result[4] = (int)((t1 - t0) / 1000);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) result[2] = abort_flag;
}

// status: one device int (the workspace status word's stand-in); result: five
// device ints.  Returns a cudaError_t value.
extern "C" int wait_timeout_probe(int* status, int* result, unsigned long long limit_ns,
                                  unsigned long long other_ns, int mode) {
  wait_timeout_probe_kernel<<<1, 64>>>(status, result, limit_ns, other_ns, mode);
  return (int)cudaGetLastError();
}
