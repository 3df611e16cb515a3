// Weight-gradient GEMM whose split-K scratch lives in a fixed device array
// owned by the library, for callers that cannot hand the library any
// device memory of its own.

#include <mutex>

#include "../../include/gpt2.h"
#include "../../include/gpt2_kernels.h"
#include "kernels.h"

using namespace gpt2k;

namespace {

// 4 Mi floats = 16 MiB on every GPU that loads this library, held until the
// process exits; every call of the entry point shares it.
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
  int* err = err_dev ? err_dev : slots.err;
  if (!err_dev && cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess) return GPT2_ERR_CUDA;
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
