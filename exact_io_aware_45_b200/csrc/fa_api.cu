// C ABI of libfa.so: argument checks, workspace layout, kernel choice.
//
// See include/fa.h for the contract. Nothing here allocates device memory;
// every launch goes to the caller's stream.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>

#include <atomic>

#include "fa.h"
#include "internal.h"

namespace fa {

static thread_local int t_launches = 0;
void count_launch(int n) { t_launches += n; }

// Wait-limit test hook (fa_debug_set_stall): kernel families with an injected
// wait and its limit in SM cycles. Process-wide; read at each launch.
static std::atomic<int> g_stall_families{0};
static std::atomic<long long> g_stall_cycles{0};
long long debug_stall_cycles(int family) {
  return (g_stall_families.load(std::memory_order_relaxed) & family)
             ? g_stall_cycles.load(std::memory_order_relaxed)
             : 0;
}

namespace {

constexpr size_t kErrBlock = 256;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool d_supported_simt(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

// Common checks of the sizes and flags. Returns FA_OK, or an error code.
fa_status check_dims(int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                     int dtype) {
  if (B < 0 || N < 0 || Hq <= 0 || Hkv <= 0 || d <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (dtype != FA_F32 && dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (!isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (!d_supported_simt(d)) return FA_ERR_UNSUPPORTED;
  // 64-bit element offsets are used everywhere; keep each tensor under 2^31
  // rows of d so that row indices fit in int.
  if ((long long)B * Hq * N >= (1ll << 31)) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

void fill_common(Problem& p, int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                 const uint8_t* mask, int dtype, void* stream) {
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.d = d;
  p.scale = scale;
  p.causal = causal;
  p.wl = -1;
  p.wr = causal ? 0 : -1;
  p.mask = mask;
  p.nb = (N + 127) / 128;
  p.Npad = p.nb * 128;
  p.dtype = dtype;
  p.stream = static_cast<cudaStream_t>(stream);
}

fa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FA_OK : FA_ERR_CUDA; }

// Mask / score modifiers of a call (fa_mods), validated. `any` is false for a
// call without modifiers (the plain entry points).
struct Mods {
  bool any = false;
  int wl = -1, wr = -1, prefix = 0;
  const int* doc = nullptr;
  float softcap = 0.f;
};

fa_status read_mods(const fa_mods* m, Mods& out) {
  out = Mods();
  if (!m) return FA_OK;
  if (m->window_left < -1 || m->window_right < -1 || m->prefix < 0) return FA_ERR_INVALID_ARG;
  if (m->doc_ids && (reinterpret_cast<uintptr_t>(m->doc_ids) & 3u)) return FA_ERR_INVALID_ARG;
  if (!isfinite(m->softcap) || m->softcap < 0.f) return FA_ERR_INVALID_ARG;
  out.wl = m->window_left;
  out.wr = m->window_right;
  out.prefix = m->prefix;
  out.doc = m->doc_ids;
  out.softcap = m->softcap;
  out.any = out.wl >= 0 || out.wr >= 0 || out.prefix > 0 || out.doc != nullptr ||
            out.softcap > 0.f;
  return FA_OK;
}

// Puts the modifiers into the problem. They run on the tensor-core kernels
// only: returns false when the caller forced the CUDA-core ones.
bool apply_mods(const Mods& m, int causal, int& path, Problem& p) {
  if (!m.any) return true;
  if (path == FA_PATH_SIMT) return false;
  path = FA_PATH_TC;
  p.wl = m.wl;
  p.wr = causal ? 0 : m.wr;
  p.prefix = m.prefix;
  p.doc = m.doc;
  p.softcap = m.softcap;
  return true;
}

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" {

const char* fa_status_string(int s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    default: return "FA_ERR_UNKNOWN";
  }
}

int fa_version(void) { return 10000; }

int fa_last_launch_count(void) { return t_launches; }

fa_status fa_debug_set_stall(int kernels, long long wait_cycles) {
  if (kernels < 0 || kernels > (FA_STALL_FWD | FA_STALL_BWD | FA_STALL_DQ))
    return FA_ERR_INVALID_ARG;
  if (kernels != 0 && (wait_cycles < 1000 || wait_cycles > 2000000000ll))
    return FA_ERR_INVALID_ARG;
  g_stall_cycles.store(kernels ? wait_cycles : 0);
  g_stall_families.store(kernels);
  return FA_OK;
}

fa_status fa_exp2_fma(const float* x, float* y, long long n, void* stream) {
  t_launches = 0;
  if (n < 0 || (n > 0 && (!x || !y))) return FA_ERR_INVALID_ARG;
  if (n > (1ll << 40)) return FA_ERR_UNSUPPORTED;
  return from_cuda(exp2_fma_eval(x, y, n, static_cast<cudaStream_t>(stream)));
}

size_t fa_fwd_workspace_size(void) { return kErrBlock; }

size_t fa_bwd_workspace_size(int B, int Hq, int N, int d) {
  if (B < 0 || Hq < 0 || N < 0 || d < 0) return 0;
  const size_t npad = (size_t)((N + 127) / 128) * 128;
  const size_t vec = align256(sizeof(float) * (size_t)B * Hq * npad);
  const size_t acc = align256(sizeof(float) * (size_t)B * Hq * N * d);
  return kErrBlock + 2 * vec + acc;
}

}  // extern "C"

namespace fa {
namespace {

fa_status fwd_impl(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                    int Hq, int Hkv, int N, int d, float scale, int causal,
                    const uint8_t* block_mask, int dtype, void* workspace, void* stream,
                    int path, const fa_mods* mods = nullptr) {
  t_launches = 0;
  Mods md;
  if (fa_status ms = read_mods(mods, md)) return ms;
  fa_status s = check_dims(B, Hq, Hkv, N, d, scale, causal, dtype);
  if (s != FA_OK) return s;
  if (path != FA_PATH_AUTO && path != FA_PATH_SIMT && path != FA_PATH_TC)
    return FA_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return FA_OK;
  if (!Q || !K || !V || !O || !LSE || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE) ||
      !aligned16(workspace))
    return FA_ERR_INVALID_ARG;
  Problem p;
  fill_common(p, B, Hq, Hkv, N, d, scale, causal, block_mask, dtype, stream);
  p.Q = Q;
  p.K = K;
  p.V = V;
  p.Oout = O;
  p.LSEout = LSE;
  p.err = static_cast<unsigned*>(workspace);
  if (!apply_mods(md, causal, path, p)) return FA_ERR_UNSUPPORTED;
  const bool tc_ok = sm100_fwd_supported(p);
  if (path == FA_PATH_TC && !tc_ok) return FA_ERR_UNSUPPORTED;
  const bool use_tc = (path == FA_PATH_TC) || (path == FA_PATH_AUTO && tc_ok);
  return from_cuda(use_tc ? sm100_fwd(p) : simt_fwd(p));
}

}  // namespace
}  // namespace fa

extern "C" {

fa_status fa_fwd_ex(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                    int Hq, int Hkv, int N, int d, float scale, int causal,
                    const uint8_t* block_mask, int dtype, void* workspace, void* stream,
                    int path) {
  return fwd_impl(Q, K, V, O, LSE, B, Hq, Hkv, N, d, scale, causal, block_mask, dtype, workspace,
                  stream, path);
}

fa_status fa_fwd_window(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                        int Hq, int Hkv, int N, int d, float scale, int causal, int window_left,
                        int window_right, const uint8_t* block_mask, int dtype, void* workspace,
                        void* stream) {
  if (window_left < -1 || window_right < -1) return FA_ERR_INVALID_ARG;
  // the window call always runs the windowed kernels, also for (-1, -1)
  fa_mods m = {window_left, window_right, 0, nullptr, 0.f};
  return fwd_impl(Q, K, V, O, LSE, B, Hq, Hkv, N, d, scale, causal, block_mask, dtype, workspace,
                  stream, FA_PATH_TC, &m);
}

fa_status fa_fwd_mod(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                     int Hq, int Hkv, int N, int d, float scale, int causal,
                     const uint8_t* block_mask, const fa_mods* mods, int dtype, void* workspace,
                     void* stream) {
  return fwd_impl(Q, K, V, O, LSE, B, Hq, Hkv, N, d, scale, causal, block_mask, dtype, workspace,
                  stream, FA_PATH_AUTO, mods);
}

fa_status fa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                 int Hq, int Hkv, int N, int d, float scale, int causal,
                 const uint8_t* block_mask, int dtype, void* workspace, void* stream) {
  return fa_fwd_ex(Q, K, V, O, LSE, B, Hq, Hkv, N, d, scale, causal, block_mask, dtype,
                   workspace, stream, FA_PATH_AUTO);
}

}  // extern "C"

namespace fa {
namespace {

enum BwdStage { kPre = 1, kMain = 2, kFinal = 4, kAll = 7 };

fa_status bwd_impl(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                   const float* LSE, void* dQ, void* dK, void* dV, int B, int Hq, int Hkv,
                   int N, int d, float scale, int causal, const uint8_t* block_mask, int dtype,
                   int grad_dtype, void* workspace, size_t workspace_bytes, void* stream,
                   int path, int stages, const int* cu = nullptr, int total = 0,
                   int deterministic = 0, const fa_mods* mods = nullptr) {
  t_launches = 0;
  Mods md;
  if (fa_status ms = read_mods(mods, md)) return ms;
  fa_status s = check_dims(B, Hq, Hkv, N, d, scale, causal, dtype);
  if (s != FA_OK) return s;
  if (grad_dtype != FA_F32 && grad_dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (path != FA_PATH_AUTO && path != FA_PATH_SIMT && path != FA_PATH_TC)
    return FA_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return FA_OK;
  if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV || !workspace)
    return FA_ERR_INVALID_ARG;
  const void* ptrs[] = {Q, K, V, O, dO, LSE, dQ, dK, dV, workspace};
  for (const void* q : ptrs)
    if (!aligned16(q)) return FA_ERR_INVALID_ARG;
  const size_t need = cu ? fa_bwd_varlen_workspace_size(B, Hq, N, total, d)
                        : fa_bwd_workspace_size(B, Hq, N, d);
  if (workspace_bytes < need) return FA_ERR_INVALID_ARG;

  Problem p;
  fill_common(p, B, Hq, Hkv, N, d, scale, causal, block_mask, dtype, stream);
  p.cu = cu;
  p.total = total;
  if (!apply_mods(md, causal, path, p)) return FA_ERR_UNSUPPORTED;
  p.Q = Q;
  p.K = K;
  p.V = V;
  p.O = O;
  p.dO = dO;
  p.LSE = LSE;
  p.dQ = dQ;
  p.dK = dK;
  p.dV = dV;
  p.grad_dtype = grad_dtype;
  char* ws = static_cast<char*>(workspace);
  p.err = reinterpret_cast<unsigned*>(ws);
  const size_t vec = align256(sizeof(float) * (size_t)B * Hq * p.Npad);
  p.Dws = reinterpret_cast<float*>(ws + kErrBlock);
  p.LSE2ws = reinterpret_cast<float*>(ws + kErrBlock + vec);
  p.dQacc = reinterpret_cast<float*>(ws + kErrBlock + 2 * vec);

  const bool tc_ok = sm100_bwd_supported(p);
  if (path == FA_PATH_TC && !tc_ok) return FA_ERR_UNSUPPORTED;
  // variable-length batches run on the tensor-core kernels only
  if (cu && (!tc_ok || path == FA_PATH_SIMT)) return FA_ERR_UNSUPPORTED;
  // Deterministic gradients: the CUDA-core kernels use no atomics already; on
  // the tensor-core path the main kernel skips dQ and the dQ kernel computes
  // it per query tile.
  const bool det_tc = deterministic && ((path == FA_PATH_TC) || (path == FA_PATH_AUTO && tc_ok));
  if (det_tc && !sm100_dq_supported(p)) return FA_ERR_UNSUPPORTED;
  p.no_dq = det_tc ? 1 : 0;
  const bool use_tc = (path == FA_PATH_TC) || (path == FA_PATH_AUTO && tc_ok);
  // The tensor-core path accumulates dQ in fp32: straight into dQ for fp32
  // gradients, into the workspace accumulator (converted by the finalize
  // stage) for bf16 gradients. The preprocess zeroes whichever it is.
  const bool use_acc = use_tc && !det_tc && sm100_bwd_uses_dq_accumulator(p);
  if (use_tc && !use_acc) p.dQacc = static_cast<float*>(dQ);
  cudaError_t e = cudaSuccess;
  if (stages & kPre) {
    e = bwd_preprocess(p, use_tc && !det_tc);
    if (e != cudaSuccess) return FA_ERR_CUDA;
  }
  if (stages & kMain) {
    e = use_tc ? sm100_bwd_main(p) : simt_bwd_main(p);
    if (e != cudaSuccess) return FA_ERR_CUDA;
    if (det_tc) {
      e = sm100_dq(p);
      if (e != cudaSuccess) return FA_ERR_CUDA;
    }
  }
  if ((stages & kFinal) && use_acc) {
    e = dq_convert(p);
    if (e != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

}  // namespace
}  // namespace fa

extern "C" {

fa_status fa_bwd_ex(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                    const float* LSE, void* dQ, void* dK, void* dV, int B, int Hq, int Hkv,
                    int N, int d, float scale, int causal, const uint8_t* block_mask,
                    int dtype, int grad_dtype, void* workspace, size_t workspace_bytes,
                    void* stream, int path) {
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, Hq, Hkv, N, d, scale, causal, block_mask,
                  dtype, grad_dtype, workspace, workspace_bytes, stream, path, kAll);
}

fa_status fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                 const float* LSE, void* dQ, void* dK, void* dV, int B, int Hq, int Hkv, int N,
                 int d, float scale, int causal, const uint8_t* block_mask, int dtype,
                 int grad_dtype, void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, Hq, Hkv, N, d, scale, causal, block_mask,
                  dtype, grad_dtype, workspace, workspace_bytes, stream, FA_PATH_AUTO, kAll);
}

#define FA_STAGE_ENTRY(name, stage)                                                            \
  fa_status name(const void* Q, const void* K, const void* V, const void* O, const void* dO,   \
                 const float* LSE, void* dQ, void* dK, void* dV, int B, int Hq, int Hkv,       \
                 int N, int d, float scale, int causal, const uint8_t* block_mask, int dtype,  \
                 int grad_dtype, void* workspace, size_t workspace_bytes, void* stream,        \
                 int path) {                                                                   \
    return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, Hq, Hkv, N, d, scale, causal,          \
                    block_mask, dtype, grad_dtype, workspace, workspace_bytes, stream, path,   \
                    stage);                                                                    \
  }

FA_STAGE_ENTRY(fa_bwd_preprocess, kPre)
FA_STAGE_ENTRY(fa_bwd_main, kMain)
FA_STAGE_ENTRY(fa_bwd_finalize, kFinal)

fa_status fa_bwd_window(const void* Q, const void* K, const void* V, const void* O,
                        const void* dO, const float* LSE, void* dQ, void* dK, void* dV, int B,
                        int Hq, int Hkv, int N, int d, float scale, int causal, int window_left,
                        int window_right, const uint8_t* block_mask, int dtype, int grad_dtype,
                        void* workspace, size_t workspace_bytes, void* stream) {
  if (window_left < -1 || window_right < -1) return FA_ERR_INVALID_ARG;
  // the window call always runs the windowed kernels, also for (-1, -1)
  fa_mods m = {window_left, window_right, 0, nullptr, 0.f};
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, Hq, Hkv, N, d, scale, causal, block_mask,
                  dtype, grad_dtype, workspace, workspace_bytes, stream, FA_PATH_TC, kAll,
                  nullptr, 0, 0, &m);
}

fa_status fa_bwd_mod(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                     const float* LSE, void* dQ, void* dK, void* dV, int B, int Hq, int Hkv,
                     int N, int d, float scale, int causal, const uint8_t* block_mask,
                     const fa_mods* mods, int dtype, int grad_dtype, void* workspace,
                     size_t workspace_bytes, void* stream) {
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, Hq, Hkv, N, d, scale, causal, block_mask,
                  dtype, grad_dtype, workspace, workspace_bytes, stream, FA_PATH_AUTO, kAll,
                  nullptr, 0, 0, mods);
}

fa_status fa_bwd_deterministic(const void* Q, const void* K, const void* V, const void* O,
                               const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                               int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                               const uint8_t* block_mask, int dtype, int grad_dtype,
                               void* workspace, size_t workspace_bytes, void* stream, int path) {
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, Hq, Hkv, N, d, scale, causal, block_mask,
                  dtype, grad_dtype, workspace, workspace_bytes, stream, path, kAll, nullptr, 0,
                  1);
}

size_t fa_bwd_varlen_workspace_size(int B, int Hq, int max_seqlen, int total, int d) {
  if (B < 0 || Hq < 0 || max_seqlen < 0 || total < 0 || d < 0) return 0;
  const size_t npad = (size_t)((max_seqlen + 127) / 128) * 128;
  const size_t vec = align256(sizeof(float) * (size_t)B * Hq * npad);
  const size_t acc = align256(sizeof(float) * (size_t)total * Hq * d);
  return kErrBlock + 2 * vec + acc;
}

}  // extern "C"

namespace fa {
namespace {

// Checks shared by the variable-length entry points (they run on the
// tensor-core kernels only: bf16, d in {64, 128}).
fa_status check_varlen(const int* cu, int B, int max_seqlen, int total, int Hq, int Hkv, int d,
                       float scale, int causal, int dtype) {
  if (B < 0 || max_seqlen < 0 || total < 0 || Hq <= 0 || Hkv <= 0 || d <= 0)
    return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0 || (causal != 0 && causal != 1)) return FA_ERR_INVALID_ARG;
  if (dtype != FA_F32 && dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (!isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (B > 0 && (!cu || (reinterpret_cast<uintptr_t>(cu) & 3u))) return FA_ERR_INVALID_ARG;
  if (total > 0 && max_seqlen == 0) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 || (d != 64 && d != 128) || !(scale > 0.f)) return FA_ERR_UNSUPPORTED;
  if ((long long)total * Hq >= (1ll << 31) || (long long)total * Hkv >= (1ll << 31) ||
      (long long)B * Hq * (((long long)max_seqlen + 127) / 128 * 128) >= (1ll << 31))
    return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

}  // namespace
}  // namespace fa

extern "C" {

fa_status fa_fwd_varlen(const void* Q, const void* K, const void* V, void* O, float* LSE,
                        const int* cu_seqlens, int B, int max_seqlen, int total, int Hq, int Hkv,
                        int d, float scale, int causal, int dtype, void* workspace,
                        void* stream) {
  t_launches = 0;
  fa_status s = check_varlen(cu_seqlens, B, max_seqlen, total, Hq, Hkv, d, scale, causal, dtype);
  if (s != FA_OK) return s;
  if (B == 0 || total == 0) return FA_OK;
  if (!Q || !K || !V || !O || !LSE || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE) ||
      !aligned16(workspace))
    return FA_ERR_INVALID_ARG;
  Problem p;
  fill_common(p, B, Hq, Hkv, max_seqlen, d, scale, causal, nullptr, dtype, stream);
  p.cu = cu_seqlens;
  p.total = total;
  p.Q = Q;
  p.K = K;
  p.V = V;
  p.Oout = O;
  p.LSEout = LSE;
  p.err = static_cast<unsigned*>(workspace);
  if (!sm100_fwd_supported(p)) return FA_ERR_UNSUPPORTED;
  return from_cuda(sm100_fwd(p));
}

fa_status fa_bwd_varlen(const void* Q, const void* K, const void* V, const void* O,
                        const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                        const int* cu_seqlens, int B, int max_seqlen, int total, int Hq, int Hkv,
                        int d, float scale, int causal, int dtype, int grad_dtype,
                        void* workspace, size_t workspace_bytes, void* stream) {
  t_launches = 0;
  fa_status s = check_varlen(cu_seqlens, B, max_seqlen, total, Hq, Hkv, d, scale, causal, dtype);
  if (s != FA_OK) return s;
  if (grad_dtype != FA_F32 && grad_dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (B == 0 || total == 0) return FA_OK;
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, Hq, Hkv, max_seqlen, d, scale, causal,
                  nullptr, dtype, grad_dtype, workspace, workspace_bytes, stream, FA_PATH_TC,
                  kAll, cu_seqlens, total);
}

fa_status fa_get_device_error(void* workspace, void* stream) {
  if (!workspace) return FA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st) !=
      cudaSuccess)
    return FA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return FA_ERR_CUDA;
  if (word == 0) return FA_OK;
  if (cudaMemsetAsync(workspace, 0, sizeof(word), st) != cudaSuccess) return FA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return FA_ERR_CUDA;
  return (word & kErrTimeout) ? FA_ERR_TIMEOUT : FA_ERR_CUDA;
}

}  // extern "C"
