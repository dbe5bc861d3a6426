// Self-check of the bounded device waits that every tensor-core kernel uses
// (mbarrier waits that give up after a fixed budget of global-timer time,
// record a timeout in the error word and let the kernel return, instead of
// spinning until the process is killed).
//
// gpt2_wait_selfcheck launches one CTA whose thread 0 waits, through that
// same routine, for an mbarrier phase that nothing completes: the wait must
// expire, the error word must then read as a timeout, and the device must
// stay usable.  Nothing faults and nothing hangs: the kernel ends on its own
// after the wait budget (2 s).

#include "tc_common.cuh"

namespace {

__global__ void wait_selfcheck_kernel(int* err, int* done) {
  __shared__ uint64_t bar;
  const uint32_t b = tc::smem_u32(&bar);
  if (threadIdx.x == 0) {
    tc::mbar_init(b, 1);  // one arrival expected; none will come
    tc::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = tc::mbar_wait(b, 0, err, 90);
    *done = ok ? 2 : 1;  // 1: the wait gave up, as it should
  }
}

}  // namespace

extern "C" int gpt2_wait_selfcheck(int* expired) {
  if (!expired) return GPT2_ERR_ARG;
  *expired = 0;
  int* err = device_error_word();
  if (!err) {
    gpt2_internal::set_error("wait_selfcheck: no device error word");
    return GPT2_ERR_CUDA;
  }
  int* done = nullptr;
  GPT2_CUDA_TRY(cudaMalloc(&done, sizeof(int)));
  cudaError_t e = cudaMemset(done, 0, sizeof(int));
  if (e == cudaSuccess) {
    wait_selfcheck_kernel<<<1, 32>>>(err, done);
    COUNT_LAUNCH(1);
    e = cudaGetLastError();
  }
  int h_done = 0;
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&h_done, done, sizeof(int), cudaMemcpyDeviceToHost);
  cudaFree(done);
  if (e != cudaSuccess) {
    gpt2_internal::set_error(std::string("wait_selfcheck: ") + cudaGetErrorString(e));
    return GPT2_ERR_CUDA;
  }
  int code = 0;
  GPT2_CUDA_TRY(cudaMemcpy(&code, err, sizeof(int), cudaMemcpyDeviceToHost));
  const int zero = 0;
  GPT2_CUDA_TRY(cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice));
  *expired = (h_done == 1 && code == 90) ? 1 : 0;
  return GPT2_OK;
}
