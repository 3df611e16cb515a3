// Weight-gradient GEMM whose split-K scratch lives in a fixed device array
// owned by the library, for callers that cannot hand the library any
// device memory of its own.

#include <mutex>

#include "../../include/gpt2.h"
#include "../../include/gpt2_kernels.h"
#include "kernels.h"

using namespace gpt2k;

namespace {

// 4 Mi floats = 16 MiB on every GPU where the entry point has run, held
// until the process exits; every call of the entry point shares it.  With
// lazy module loading (the CUDA default since 12.2) the driver places the
// array on a device when the first call there looks up its address, so
// that first call needs 16 MiB of free device memory.
static __device__ __align__(256) float g_wgrad_scratch[GPT2K_NOALLOC_SCRATCH_FLOATS];
static __device__ __align__(256) int g_wgrad_err[1];

struct DeviceSlots {
  bool ready = false;
  float* scratch = nullptr;  // device address of g_wgrad_scratch on that device
  int* err = nullptr;
};

constexpr int kMaxDevices = 64;
std::mutex g_mu;
DeviceSlots g_slots[kMaxDevices];

// Once per device, with that device current: the host-side names of the two
// arrays are stand-ins, so their device addresses are looked up here.
int device_slots(DeviceSlots* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GPT2_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceSlots& s = g_slots[dev];
  if (!s.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_wgrad_scratch) != cudaSuccess || !p) return GPT2_ERR_CUDA;
    s.scratch = static_cast<float*>(p);
    p = nullptr;
    if (cudaGetSymbolAddress(&p, g_wgrad_err) != cudaSuccess || !p) return GPT2_ERR_CUDA;
    s.err = static_cast<int*>(p);
    s.ready = true;
  }
  *out = s;
  return GPT2_OK;
}

}  // namespace

namespace gpt2k {

// Error bits that calls made with err_dev = NULL left in the private error
// word of the current device, read and cleared (synchronous); 0 when the
// entry point has not been set up on this device.
int noalloc_take_error() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  int* err = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_slots[dev].ready) return 0;
    err = g_slots[dev].err;
  }
  int e = 0;
  if (cudaMemcpy(&e, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return 0;
  cudaMemset(err, 0, sizeof(int));
  return e;
}

}  // namespace gpt2k

extern "C" int gpt2k_gemm_wgrad_noalloc(void* stream, int M, int N, int K, const void* A,
                                        long lda, const void* B, long ldb, float alpha,
                                        float* out32, long ldo32, int max_splits, int* err_dev) {
  if (M < 1 || N < 1 || K < 1 || max_splits < 1 || max_splits > 8 || !A || !B || !out32)
    return GPT2_ERR_ARG;
  if ((size_t)max_splits * (size_t)M * (size_t)N > GPT2K_NOALLOC_SCRATCH_FLOATS)
    return GPT2_ERR_ARG;  // the partial sums would not fit in the fixed scratch array
  DeviceSlots slots;
  const int st = device_slots(&slots);
  if (st != GPT2_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Without err_dev the expiry bit goes to the private word, which keeps
  // accumulating until gpt2k_take_error reads and clears it.
  int* err = err_dev ? err_dev : slots.err;
  GemmArgs g{};
  g.M = M; g.N = N; g.K = K;
  g.A = static_cast<const act_t*>(A); g.lda = lda; g.a_mn = 1;
  g.B = static_cast<const act_t*>(B); g.ldb = ldb; g.b_mn = 1;
  g.epi = EPI_F32_ACC;
  g.alpha = alpha;
  g.out32 = out32; g.ldo32 = ldo32;
  g.split_ws = slots.scratch;
  g.split_ws_floats = (size_t)max_splits * M * N;
  g.max_splits = max_splits;
  const cudaError_t e = gemm(g, s, err);
  if (e == cudaSuccess) return GPT2_OK;
  return e == cudaErrorInvalidValue ? GPT2_ERR_ARG : GPT2_ERR_CUDA;
}
