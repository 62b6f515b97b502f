// The bounded poll behind every wait inside the kernels (mbarrier phases,
// flags written by other CTAs).  No wait may spin forever: after `limit`
// nanoseconds of the caller's clock, or once another role of the CTA has
// raised the abort flag, it gives up and the caller reports MOE_DEV_TIMEOUT.
//
// Written without any CUDA construct so that the same template also compiles
// for the host, where a test drives it with a fake clock and condition.
#pragma once

#ifdef __CUDACC__
#define MOE_HOST_DEVICE __host__ __device__ __forceinline__
#else
#define MOE_HOST_DEVICE inline
#endif

namespace moe {

// Polls ready() until it returns true (returns true).  After the first miss
// it reads the clock once; then, every `every` polls (a power of two), it
// returns false if *abort_flag (may be null) is set or if more than `limit`
// has elapsed since that first reading.  pause() runs between polls.
template <class Ready, class Now, class Pause>
MOE_HOST_DEVICE bool bounded_poll(Ready ready, Now now, Pause pause, const volatile int* abort_flag,
                                  unsigned long long limit, unsigned every) {
  if (ready()) return true;
  const unsigned long long t0 = now();
  for (unsigned i = 1;; ++i) {
    pause();
    if (ready()) return true;
    if ((i & (every - 1u)) == 0u) {
      if (abort_flag != nullptr && *abort_flag) return false;
      if (now() - t0 > limit) return false;
    }
  }
}

}  // namespace moe
