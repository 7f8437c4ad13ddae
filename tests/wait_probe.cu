// wait_probe.cu -- test helper, built by tests/test_gpu_bounded_wait.py: a kernel
// whose mbarrier wait can never complete (nothing ever arrives on the barrier),
// compiled from the library's own device header so that it exercises the same
// bounded wait the library's kernels use.  The wait must give up after
// IC_WAIT_NS, raise the CTA's abort flag (a second role then gives up at once),
// record its error code and return, leaving the context usable.
#include "../sparse_attention_indexer_sum_b200/csrc/ic_device.cuh"

__global__ void wait_probe_kernel(int* result) {
  __shared__ alignas(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ic::mbar_init(ic::smem_u32(&bar), 1);
    abort_flag = 0;
    ic::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = ic::mbar_wait(ic::smem_u32(&bar), 0, &abort_flag, ic::kErrTimeoutEpilogue);
    result[0] = ok ? 1 : 0;
  } else if (threadIdx.x == 32) {
    // another role waiting on the same barrier: released by the abort flag
    const bool ok = ic::mbar_wait(ic::smem_u32(&bar), 0, &abort_flag, ic::kErrTimeoutMma);
    result[1] = ok ? 1 : 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) result[2] = abort_flag;
}

extern "C" int wait_probe_launch(int* result, void* stream) {
  wait_probe_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(result);
  return static_cast<int>(cudaGetLastError());
}

extern "C" int wait_probe_error_word() {
  int v = -1;
  if (cudaMemcpyFromSymbol(&v, ic::g_dev_error, sizeof(int)) != cudaSuccess) return -1;
  return v;
}
