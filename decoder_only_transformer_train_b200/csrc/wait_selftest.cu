// Self-test of the bounded mbarrier waits that every pipelined kernel of this library uses
// (sm100.cuh): a wait that nothing will ever end must give up after its limit, record
// GPT2_ERR_TIMEOUT in the device error word, let a copy still in flight land, and return,
// leaving the context usable.  No GPU fault, trap or endless loop is involved: the waits
// poll with a time limit taken from %globaltimer.
#include "gpt2_b200.h"
#include "sm100.cuh"
#include "kernels.h"

namespace {

// Warp 0, lane 0: starts a 16-byte bulk copy, then waits alone on a barrier nobody arrives
// on (mbar_wait); after giving up it waits for its copy to land (mbar_drain).
// Warp 1: all 32 lanes wait together on another barrier nobody arrives on (mbar_wait_warp);
// the warp vote makes them leave together, which the __syncwarp after it relies on.
// status[0], status[1]: 1 if the wait of warp 0 / warp 1 succeeded, 0 if it gave up.
__global__ void __launch_bounds__(64) bounded_wait_selftest_kernel(const uint4* __restrict__ src, uint64_t limit_ns,
                                                                   int* __restrict__ status) {
  __shared__ __align__(16) uint4 buf;
  __shared__ __align__(8) uint64_t bars[3];
  __shared__ int abort_word;
  volatile int* abort_flag = &abort_word;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars[2], 16);
      bulk_load(&buf, src, 16, &bars[2]);
      const bool ok = mbar_wait(&bars[0], 0, abort_flag, limit_ns);
      if (!ok) mbar_drain(&bars[2], 0);
      status[0] = ok ? 1 : 0;
    }
  } else {
    const bool ok = mbar_wait_warp(&bars[1], 0, abort_flag, limit_ns);
    __syncwarp();
    if (lane == 0) status[1] = ok ? 1 : 0;
  }
  __syncthreads();
}

}  // namespace

extern "C" int gpt2op_bounded_wait_selftest(void* stream, int64_t limit_ns, const void* src16, int* status) {
  if (src16 == nullptr || status == nullptr) return GPT2_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(src16) % 16 || reinterpret_cast<uintptr_t>(status) % 4) return GPT2_ERR_ARG;
  if (limit_ns <= 0 || limit_ns > 1000000000ll) return GPT2_ERR_ARG;
  bounded_wait_selftest_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint4*>(src16), (uint64_t)limit_ns, status);
  note_kernel_launches(1);
  return cudaGetLastError() == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
}
