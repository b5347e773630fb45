// Internal interface between the C ABI (fa_api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

// Everything a launch needs, validated by the ABI layer.
struct Problem {
  // inputs
  const void* Q = nullptr;
  const void* K = nullptr;
  const void* V = nullptr;
  const void* O = nullptr;      // forward output (backward input)
  const void* dO = nullptr;
  const float* LSE = nullptr;   // forward LSE (backward input)
  // outputs
  void* Oout = nullptr;
  float* LSEout = nullptr;
  void* dQ = nullptr;
  void* dK = nullptr;
  void* dV = nullptr;
  // sizes and options
  int B = 0, Hq = 0, Hkv = 0, N = 0, d = 0;
  float scale = 1.f;
  int causal = 0;
  // sliding window: visible keys j of query i satisfy i - wl <= j <= i + wr
  // (-1: unbounded); the launchers apply the causal flag as wr = 0 on top
  int wl = -1, wr = -1;
  // prefix LM: keys below `prefix` are visible to every query whatever the
  // right bound says (0: none); doc: [N] non-decreasing per-token document ids
  // (a query sees only its own document), or null
  int prefix = 0;
  const int* doc = nullptr;
  // soft-capping score modifier: scores x = scale * q.k become
  // softcap * tanh(x / softcap) (0: off)
  float softcap = 0.f;
  const uint8_t* mask = nullptr;  // [nb * nb] or null
  int nb = 0;                     // ceil(N / 128)
  int dtype = 0;                  // 0 f32, 1 bf16
  int grad_dtype = 0;
  // workspace pieces
  unsigned* err = nullptr;        // device error word
  float* Dws = nullptr;           // [B*Hq][Npad]
  float* LSE2ws = nullptr;        // [B*Hq][Npad]  LSE * log2(e), +inf where empty
  float* dQacc = nullptr;         // [B*Hq][N][d]
  int Npad = 0;
  // variable-length batch: sequence b is rows cu[b] .. cu[b+1]-1 of packed
  // [total][H][d] tensors (LSE [Hq][total]); N is then the longest length
  const int* cu = nullptr;
  int total = 0;
  // backward main kernel: skip dQ (computed by the deterministic dQ kernel)
  int no_dq = 0;
  cudaStream_t stream = nullptr;
};

// Error-word bits set by kernels.
enum : unsigned { kErrTimeout = 1u, kErrBounds = 2u };

// Kernel families of the wait-limit test hook (fa_debug_set_stall).
enum : int { kStallFwd = 1, kStallBwd = 2, kStallDq = 4 };
// Wait limit (SM cycles) of the injected wait of the given family, or 0 when
// the hook is off for it.
long long debug_stall_cycles(int family);

// Counts launches made by the current ABI call (thread-local).
void count_launch(int n = 1);

// CUDA-core kernels (fp32 arithmetic). simt_kernels.cu
cudaError_t simt_fwd(const Problem& p);
cudaError_t bwd_preprocess(const Problem& p, bool zero_dq_accumulator);
cudaError_t simt_bwd_main(const Problem& p);
cudaError_t dq_convert(const Problem& p);

// tcgen05 / TMA kernels for sm_100a. sm100_fwd.cu, sm100_bwd.cu
bool sm100_fwd_supported(const Problem& p);
cudaError_t sm100_fwd(const Problem& p);
// Evaluates the forward kernel's FMA-pipe exp2 on n floats (diagnostic).
cudaError_t exp2_fma_eval(const float* x, float* y, long long n, cudaStream_t stream);
bool sm100_bwd_supported(const Problem& p);
bool sm100_bwd_uses_dq_accumulator(const Problem& p);
cudaError_t sm100_bwd_main(const Problem& p);
// Deterministic dQ (no atomics): one CTA per query tile. sm100_dq.cu
bool sm100_dq_supported(const Problem& p);
cudaError_t sm100_dq(const Problem& p);

}  // namespace fa
