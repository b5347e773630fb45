// fa_bwd_noalloc: the backward pass for callers that cannot allocate device
// memory.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: code
// running inside another runtime's memory pool that forbids side allocations,
// plugins whose host owns every device buffer, or latency-critical paths
// where an allocation could block or fragment the pool. For them the
// backward's scratch (the per-row D = rowsum(dO * O) and LSE * log2(e)
// vectors) lives in a fixed array in this library's device image instead of
// a caller workspace. The kernels are the same ones fa_bwd launches.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "fa.h"
#include "internal.h"

namespace fa {
namespace {

// Largest B * Hq * ceil(N / 128) * 128 the array can serve (rows of D and of
// the log2-scaled LSE, one float each): 2 x 4 MiB plus a 256-byte block for
// the fallback error word, about 8 MiB per GPU that loads the library.
constexpr size_t kMaxRows = size_t(1) << 20;
constexpr size_t kHead = 256;
constexpr size_t kBytes = kHead + 2 * kMaxRows * sizeof(float);

// Device-resident scratch, shared by every call on a device. Host code sees
// only a host-side stand-in under this name; the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_scratch[kBytes];

constexpr int kMaxDevices = 64;

// Device address of g_scratch on the current device, looked up once per
// device (with that device current) and cached.
cudaError_t scratch_address(unsigned char** out) {
  static std::mutex mu;
  static unsigned char* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<unsigned char*>(p);
  }
  *out = addr[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" fa_status fa_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O,
                                    const void* dO, const float* LSE, float* dQ, float* dK,
                                    float* dV, int B, int Hq, int Hkv, int N, int d, float scale,
                                    int causal, const uint8_t* block_mask, int dtype,
                                    unsigned* device_error, void* stream) {
  if (B < 0 || N < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if ((causal != 0 && causal != 1) || (dtype != FA_F32 && dtype != FA_BF16) || !isfinite(scale))
    return FA_ERR_INVALID_ARG;
  if (d != 16 && d != 32 && d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return FA_OK;
  const size_t npad = (size_t)((N + 127) / 128) * 128;
  if ((size_t)B * Hq * npad > kMaxRows) return FA_ERR_UNSUPPORTED;  // beyond the fixed array
  const void* ptrs[] = {Q, K, V, O, dO, LSE, dQ, dK, dV};
  for (const void* q : ptrs)
    if (!q || !aligned16(q)) return FA_ERR_INVALID_ARG;
  if (device_error && (reinterpret_cast<uintptr_t>(device_error) & 3u)) return FA_ERR_INVALID_ARG;

  unsigned char* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return FA_ERR_CUDA;

  Problem p;
  p.Q = Q;
  p.K = K;
  p.V = V;
  p.O = O;
  p.dO = dO;
  p.LSE = LSE;
  p.dQ = dQ;
  p.dK = dK;
  p.dV = dV;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.d = d;
  p.scale = scale;
  p.causal = causal;
  p.mask = block_mask;
  p.nb = (N + 127) / 128;
  p.Npad = p.nb * 128;
  p.dtype = dtype;
  p.grad_dtype = FA_F32;
  p.stream = static_cast<cudaStream_t>(stream);
  const size_t rows = (size_t)B * Hq * npad;
  p.Dws = reinterpret_cast<float*>(scratch + kHead);
  p.LSE2ws = p.Dws + rows;
  // fp32 gradients need no separate dQ accumulator: a kernel family that
  // accumulates dQ does so in dQ itself, which the preprocess zeroes.
  p.dQacc = dQ;
  p.err = device_error ? device_error : reinterpret_cast<unsigned*>(scratch);
  if (!device_error && cudaMemsetAsync(p.err, 0, sizeof(unsigned), p.stream) != cudaSuccess)
    return FA_ERR_CUDA;

  const bool use_tc = sm100_bwd_supported(p);
  if (use_tc && sm100_bwd_uses_dq_accumulator(p)) return FA_ERR_UNSUPPORTED;
  if (bwd_preprocess(p, use_tc) != cudaSuccess) return FA_ERR_CUDA;
  if ((use_tc ? sm100_bwd_main(p) : simt_bwd_main(p)) != cudaSuccess) return FA_ERR_CUDA;
  return FA_OK;
}
