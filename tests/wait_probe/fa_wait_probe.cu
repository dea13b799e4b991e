// Test-only variant of the library: every entry point of fa_api.cu, compiled
// with a short bound on device pipeline waits (the test passes
// -DFA_WAIT_TIMEOUT_NS), plus one probe kernel whose wait can never be
// satisfied.  It shows, on a GPU and without any fault, that an expired wait
// ends the kernel, lets the CTA's other warps leave through the abort flag,
// frees the CTA's tensor memory, and is reported by fa_get_device_error() as
// FA_ERR_TIMEOUT -- after which the same context runs the library's kernels
// normally.  Not part of the product library.
#include "../../exact_io_aware_95_b200/csrc/fa_api.cu"

namespace fa {

// Delay of the second waiter, so that it is still inside its own time limit
// when the first waiter's limit expires.
constexpr uint64_t kProbeDelayNs = 5000000ull;

// One CTA of 64 threads, set up like the library's kernels (mbarriers and an
// abort flag in shared memory; warp 1 allocates tensor memory).  Warp 0 waits
// on `never`, an mbarrier that nothing arrives on, with the library's bounded
// wait.  Warp 1, after a bounded delay, waits on `also_never`; it must leave
// because warp 0 raised the abort flag.  Then the common teardown frees the
// tensor memory.  rec[0..4]: warp 0's result and elapsed ns, warp 1's result
// and elapsed ns, the abort flag warp 1 saw.
__global__ void __launch_bounds__(64, 1) fa_wait_probe_kernel(long long* rec) {
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_word;
  const int warp = threadIdx.x >> 5;
  const uint32_t never = smem_u32(&bars[0]), also_never = smem_u32(&bars[1]);
  volatile int* abort_flag = &abort_word;
  if (threadIdx.x == 0) {
    mbar_init(never, 1);
    mbar_init(also_never, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint64_t t0 = global_timer_ns();
  if (warp == 0) {
    const bool ok = mbar_wait(never, 0, abort_flag);
    if (threadIdx.x == 0) {
      rec[0] = ok;
      rec[1] = static_cast<long long>(global_timer_ns() - t0);
    }
  } else {
    while (global_timer_ns() - t0 < kProbeDelayNs) {
    }
    const bool ok = mbar_wait(also_never, 0, abort_flag);
    if (threadIdx.x == 32) {
      rec[2] = ok;
      rec[3] = static_cast<long long>(global_timer_ns() - t0);
      rec[4] = *abort_flag;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_slot, 32);
  }
}

}  // namespace fa

extern "C" fa_status fa_wait_probe(long long* rec, void* stream) {
  if (!rec) return FA_ERR_INVALID_ARG;
  fa::fa_wait_probe_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(rec);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

extern "C" unsigned long long fa_wait_probe_limit_ns(void) { return FA_WAIT_TIMEOUT_NS; }
extern "C" unsigned long long fa_wait_probe_delay_ns(void) { return fa::kProbeDelayNs; }
