/*
 * fa.h -- C ABI of the exact, IO-aware tiled attention library (libfa.so).
 *
 * What is computed (FlashAttention pages: "FlashAttention" lesson by Pranay
 * Mahendrakar, Researcher section "The problem being solved" and "Online
 * softmax"; paper summary "FlashAttention: Fast and Memory-Efficient Exact
 * Attention with IO-Awareness", "Core Idea"):
 *
 *   for every batch b and query head h, with KV head hk = h / (Hq / Hkv),
 *     S   = scale * Q[b,h] K[b,hk]^T                  (N x N, never stored)
 *     S_ij = -inf where key j is not visible to query i
 *     O[b,h]   = softmax(S) V[b,hk]                    (row-wise softmax)
 *     LSE[b,h] = per-row natural-log logsumexp of S    (the saved statistic)
 *
 * Key j is visible to query i iff (causal == 0 or j <= i) and (block_mask ==
 * NULL or block_mask[(i/128) * nb + j/128] != 0), nb = ceil(N/128). A row with
 * no visible key gets O = 0 and LSE = -inf. The causal flag follows the
 * lesson's Developer section ("Common mistakes": pass the flag instead of a
 * dense N x N mask); the 128 x 128 block mask is the block-sparse extension of
 * the paper summary ("Key Method Details"); grouped KV heads are the
 * multi-query / grouped-query support of the glossary page ("FlashAttention-2
 * Improvements").
 *
 * The backward pass recomputes P on chip from Q, K and LSE (paper summary,
 * "Core Idea" item 3) and returns
 *   dV = P^T dO,  dP = dO V^T,  D_i = sum_k dO_ik O_ik,  dS = P * (dP - D),
 *   dQ = scale * dS K,  dK = scale * dS^T Q,
 * with dK and dV summed over the query heads that share a KV head.
 *
 * Layout: every tensor is contiguous row-major. Q, O, dO, dQ are [B, Hq, N, d];
 * K, V, dK, dV are [B, Hkv, N, d]; LSE is float [B, Hq, N]. All tensor
 * pointers are DEVICE pointers, 16-byte aligned. Outputs are fully
 * overwritten (dK and dV are not accumulated into). The caller owns every
 * buffer, including the workspace; the library allocates no device memory.
 * Every entry point is asynchronous on `stream` (a cudaStream_t passed as
 * void*; NULL = the legacy default stream) except fa_get_device_error, which
 * synchronises that stream.
 *
 * Errors: argument checks run on the host before any launch and return
 * FA_ERR_INVALID_ARG (malformed) or FA_ERR_UNSUPPORTED (well-formed but not
 * implemented: e.g. fp32 inputs with the tensor-core path). A failed launch
 * returns FA_ERR_CUDA. Every wait inside a kernel is bounded; a wait that runs
 * out sets a bit in the workspace's error word, the kernel returns without
 * faulting, and fa_get_device_error reports FA_ERR_TIMEOUT. While the word is
 * set, later tensor-core launches on the same workspace return without work
 * (their outputs are then undefined) until fa_get_device_error clears it. The
 * library never traps and never resets the device.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,
  FA_ERR_UNSUPPORTED = 2,
  FA_ERR_CUDA = 3,
  FA_ERR_TIMEOUT = 4
} fa_status;

/* Element types of Q, K, V, O, dO (dtype) and of dQ, dK, dV (grad_dtype). */
typedef enum { FA_F32 = 0, FA_BF16 = 1 } fa_dtype;

/* Kernel family: AUTO picks the tcgen05 tensor-core kernels for bf16 with
 * d in {64, 128} and the fp32 CUDA-core kernels otherwise; SIMT forces the
 * CUDA-core kernels (fp32 arithmetic for any supported dtype); TC forces the
 * tensor-core kernels (FA_ERR_UNSUPPORTED where they do not apply). */
typedef enum { FA_PATH_AUTO = 0, FA_PATH_SIMT = 1, FA_PATH_TC = 2 } fa_path;

/* Human-readable name of a status code (static string, never NULL). */
const char* fa_status_string(int status);

/* ABI version: major * 10000 + minor * 100 + patch. */
int fa_version(void);

/* Bytes of workspace fa_fwd needs: the 256-byte error-word block (the
 * backward's workspace starts with the same block and may serve both). */
size_t fa_fwd_workspace_size(void);

/* Bytes of workspace fa_bwd needs: the error-word block, D and the
 * log2-scaled LSE (float [B*Hq][ceil(N/128)*128] each) and the fp32 dQ
 * accumulator (float [B*Hq][N][d]). Returns 0 for negative sizes. */
size_t fa_bwd_workspace_size(int B, int Hq, int N, int d);

/*
 * Forward pass. Writes O (dtype) and LSE (float, natural log of the scaled
 * scores, -inf for rows with no visible key).
 *   Q [B,Hq,N,d], K and V [B,Hkv,N,d] (dtype); O [B,Hq,N,d] (dtype);
 *   LSE [B,Hq,N] float; scale: the softmax scale (1/sqrt(d) in the pages);
 *   causal: 0 or 1; block_mask: NULL or device uint8 [nb*nb];
 *   workspace: >= fa_fwd_workspace_size() bytes, device, its first 256 bytes
 *   zeroed once before first use. That block holds the error word (which
 *   fa_get_device_error clears) and, for the persistent form of the kernel, a
 *   work-queue counter that each launch leaves at zero again. A workspace
 *   serves one launch at a time: launches that may overlap on the GPU need
 *   workspaces of their own.
 * Supported: d in {16, 32, 64, 128}; Hq % Hkv == 0; N >= 0, B >= 0 (an empty
 * problem launches nothing and returns FA_OK).
 */
fa_status fa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE,
                 int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                 const uint8_t* block_mask, int dtype, void* workspace, void* stream);

/* fa_fwd with an explicit kernel family (fa_path). */
fa_status fa_fwd_ex(const void* Q, const void* K, const void* V, void* O, float* LSE,
                    int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                    const uint8_t* block_mask, int dtype, void* workspace, void* stream,
                    int path);

/*
 * Backward pass: dQ, dK, dV (grad_dtype) from Q, K, V, O, dO (dtype) and the
 * forward's LSE. scale, causal and block_mask must be the forward's.
 * workspace: >= fa_bwd_workspace_size(B, Hq, N, d) bytes of device memory
 * (error word zeroed once before first use; the rest is scratch, overwritten).
 * Runs three stages in order on `stream`: fa_bwd_preprocess, fa_bwd_main,
 * fa_bwd_finalize.
 */
fa_status fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                 const float* LSE, void* dQ, void* dK, void* dV,
                 int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                 const uint8_t* block_mask, int dtype, int grad_dtype,
                 void* workspace, size_t workspace_bytes, void* stream);

/* fa_bwd with an explicit kernel family (fa_path). */
fa_status fa_bwd_ex(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                    const float* LSE, void* dQ, void* dK, void* dV,
                    int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                    const uint8_t* block_mask, int dtype, int grad_dtype,
                    void* workspace, size_t workspace_bytes, void* stream, int path);

/*
 * The three stages of fa_bwd, exposed so that each kernel can be timed on
 * its own. They take fa_bwd_ex's arguments and must be called in this order
 * with the same arguments and workspace.
 *   preprocess: D_i = sum_k dO_ik O_ik and LSE * log2(e) into the workspace
 *               (rows with LSE = -inf become +inf, so their P is 0); zeroes
 *               the dQ accumulator when the main stage uses one.
 *   main:       recomputes P tile by tile; writes dK, dV and accumulates dQ.
 *   finalize:   converts the fp32 dQ accumulator to dQ (no launch when the
 *               main stage wrote dQ directly).
 */
fa_status fa_bwd_preprocess(const void* Q, const void* K, const void* V, const void* O,
                            const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                            int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                            const uint8_t* block_mask, int dtype, int grad_dtype,
                            void* workspace, size_t workspace_bytes, void* stream, int path);
fa_status fa_bwd_main(const void* Q, const void* K, const void* V, const void* O,
                      const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                      int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                      const uint8_t* block_mask, int dtype, int grad_dtype,
                      void* workspace, size_t workspace_bytes, void* stream, int path);
fa_status fa_bwd_finalize(const void* Q, const void* K, const void* V, const void* O,
                          const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                          int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                          const uint8_t* block_mask, int dtype, int grad_dtype,
                          void* workspace, size_t workspace_bytes, void* stream, int path);

/*
 * Sliding-window (local) attention: a mask modifier on top of the causal flag
 * and the block mask, in the spirit of the lesson's FlexAttention note (one
 * tiled kernel, many masks; Researcher section, "Version lineage"). Key j is
 * visible to query i iff
 *   (window_left  < 0 or j >= i - window_left) and
 *   (window_right < 0 or j <= i + window_right) and (causal == 0 or j <= i)
 * and the block mask allows it; -1 means unbounded (the causal flag wins over
 * window_right). Key tiles wholly outside the window are skipped, partly
 * covered ones masked element by element. Same arguments, layouts and
 * workspace rules as fa_fwd / fa_bwd otherwise; the backward must get the
 * forward's window. Tensor-core kernels only (bf16, d in {64, 128},
 * scale > 0): FA_ERR_UNSUPPORTED otherwise; FA_ERR_INVALID_ARG for a bound
 * below -1.
 */
fa_status fa_fwd_window(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                        int Hq, int Hkv, int N, int d, float scale, int causal, int window_left,
                        int window_right, const uint8_t* block_mask, int dtype, void* workspace,
                        void* stream);

fa_status fa_bwd_window(const void* Q, const void* K, const void* V, const void* O,
                        const void* dO, const float* LSE, void* dQ, void* dK, void* dV, int B,
                        int Hq, int Hkv, int N, int d, float scale, int causal, int window_left,
                        int window_right, const uint8_t* block_mask, int dtype, int grad_dtype,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * Mask and score modifiers: one tiled kernel, many masks (the lesson's
 * Researcher section, "Beyond hand-written kernels", on FlexAttention's
 * mask_mod and score_mod).
 * With modifiers, key j is visible to query i iff lo(i) <= j <= hi(i) and the
 * block mask allows the pair, where
 *   hi(i) = min(right(i), last row of i's document),
 *   lo(i) = max(window_left >= 0 ? i - window_left : 0, first row of i's document),
 *   right(i) = N - 1 without a right bound, else max(i + r, prefix - 1) with
 *   r = 0 under the causal flag (it wins over window_right), window_right
 *   otherwise.
 * Fields:
 *   window_left, window_right: sliding-window bounds, -1 = unbounded;
 *   prefix: >= 0; the first `prefix` keys are visible to every query whatever
 *     the right bound says (with the causal flag: a prefix language model, the
 *     prefix attending to itself in both directions);
 *   doc_ids: NULL, or device int32 [N], 4-byte aligned, one document id per
 *     token, non-decreasing (documents packed back to back; shared by every
 *     batch and head): a query sees only keys of its own document. Ids that
 *     are not sorted give wrong results but no access outside the array;
 *   softcap: >= 0; 0 = off. A score modifier (FlexAttention's score_mod):
 *     every score x = scale * q.k becomes softcap * tanh(x / softcap) before
 *     the mask and the softmax; the backward applies the chain rule
 *     d/dx = 1 - tanh^2(x / softcap). LSE is the logsumexp of the capped
 *     scores. Not combined with variable-length batches.
 * The backward must get the forward's modifiers. Tiles a query tile cannot
 * see are skipped; tiles it sees whole run unmasked; the rest are masked per
 * element. Tensor-core kernels only (dtype bf16, d in {64, 128}, scale > 0):
 * FA_ERR_UNSUPPORTED otherwise; FA_ERR_INVALID_ARG for a bound below -1, a
 * negative prefix, a misaligned doc_ids or a negative or non-finite softcap. mods == NULL, or all fields off,
 * is fa_fwd / fa_bwd.
 */
typedef struct {
  int window_left;
  int window_right;
  int prefix;
  const int* doc_ids;
  float softcap;
} fa_mods;

fa_status fa_fwd_mod(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                     int Hq, int Hkv, int N, int d, float scale, int causal,
                     const uint8_t* block_mask, const fa_mods* mods, int dtype, void* workspace,
                     void* stream);

fa_status fa_bwd_mod(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                     const float* LSE, void* dQ, void* dK, void* dV, int B, int Hq, int Hkv,
                     int N, int d, float scale, int causal, const uint8_t* block_mask,
                     const fa_mods* mods, int dtype, int grad_dtype, void* workspace,
                     size_t workspace_bytes, void* stream);

/*
 * fa_bwd with run-to-run identical gradients. fa_bwd adds the dQ partials of
 * different key tiles with fp32 reduce-adds whose order depends on
 * scheduling, so its dQ can differ in the last bits between runs (dK, dV
 * and the forward are identical run to run). Here the main kernel skips dQ
 * and a second kernel computes it per 128-row query tile, summing the key
 * tiles in a fixed order in TMEM: 3 more matrix products per (query tile,
 * key tile) pair (S, dP, dQ), so about 60 % more backward work. Arguments,
 * workspace and errors as fa_bwd_ex (path: FA_PATH_*; the CUDA-core kernels
 * are deterministic already). Not for variable-length batches.
 */
fa_status fa_bwd_deterministic(const void* Q, const void* K, const void* V, const void* O,
                               const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                               int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                               const uint8_t* block_mask, int dtype, int grad_dtype,
                               void* workspace, size_t workspace_bytes, void* stream, int path);

/*
 * Variable-length (padding-free) batches. The glossary page ("Sequence Length
 * Flexibility") names arbitrary sequence lengths without padding; these entry
 * points take B sequences packed back to back:
 *   Q, O, dO, dQ: [total][Hq][d]; K, V, dK, dV: [total][Hkv][d];
 *   LSE: float [Hq][total];
 *   cu_seqlens: device int32 [B + 1], cu_seqlens[0] = 0, non-decreasing,
 *   cu_seqlens[B] = total; sequence b is rows cu_seqlens[b] .. cu_seqlens[b+1]-1
 *   and attends only to itself (the causal flag is applied per sequence);
 *   max_seqlen >= every length (it sizes the grid).
 * Offsets are clamped to [0, total] on the device and a sequence longer than
 * max_seqlen is cut to it, so inconsistent offsets give wrong results but no
 * access outside the tensors. Tensor-core kernels only: dtype bf16, d in
 * {64, 128}, scale > 0 (FA_ERR_UNSUPPORTED otherwise); no block mask. The
 * workspace rules are those of fa_fwd / fa_bwd, with
 * fa_bwd_varlen_workspace_size for the backward.
 */
fa_status fa_fwd_varlen(const void* Q, const void* K, const void* V, void* O, float* LSE,
                        const int* cu_seqlens, int B, int max_seqlen, int total, int Hq, int Hkv,
                        int d, float scale, int causal, int dtype, void* workspace,
                        void* stream);

fa_status fa_bwd_varlen(const void* Q, const void* K, const void* V, const void* O,
                        const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                        const int* cu_seqlens, int B, int max_seqlen, int total, int Hq, int Hkv,
                        int d, float scale, int causal, int dtype, int grad_dtype,
                        void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace fa_bwd_varlen needs: the error-word block, D and the
 * log2-scaled LSE (float [B*Hq][ceil(max_seqlen/128)*128] each) and the fp32
 * dQ accumulator (float [total][Hq][d]). Returns 0 for negative sizes. */
size_t fa_bwd_varlen_workspace_size(int B, int Hq, int max_seqlen, int total, int d);

/*
 * fa_bwd_noalloc -- the backward pass for callers that cannot allocate.
 *
 * No passage of the FlashAttention pages corresponds to this entry point; it
 * exists for deployment. Some callers cannot call cudaMalloc or provide a
 * workspace buffer: code running under an allocator that owns all device
 * memory and forbids side allocations, plugins whose host hands them only
 * the tensors, or paths where an allocation could block or fragment a
 * memory pool. This entry point computes what fa_bwd computes with fp32
 * gradients (same kernels), but its scratch -- the per-row D = rowsum(dO * O)
 * and LSE * log2(e) vectors -- lives in a fixed array inside libfa.so's
 * device image (about 8 MiB, held by every GPU that loads the library until
 * the process exits). It allocates nothing and calls no allocating routine.
 *
 * Arguments as fa_bwd, except: dQ, dK, dV are float (fp32 gradients only);
 * there is no workspace; device_error is NULL or a caller-owned device word
 * (4-byte aligned) into which kernels OR a non-zero value if a bounded wait
 * runs out (the caller zeroes it; with NULL a word inside the fixed array is
 * used and cleared at each call, so timeouts are then not observable).
 *
 * Limits: B * Hq * ceil(N / 128) * 128 must not exceed 1,048,576 rows
 * (FA_ERR_UNSUPPORTED otherwise, before anything is launched).
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it; make that first call before any CUDA graph
 * capture. The cached address is not looked up again, so fa_bwd_noalloc is
 * not supported after cudaDeviceReset in the same process (the reset unloads
 * the device image and the array may come back elsewhere). Every call on a device shares the one array and leaves its
 * contents behind; calls whose kernels overlap on the GPU (different streams
 * without ordering, or several host threads) race on it and must be ordered
 * by the caller.
 */
fa_status fa_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O,
                         const void* dO, const float* LSE, float* dQ, float* dK, float* dV,
                         int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                         const uint8_t* block_mask, int dtype, unsigned* device_error,
                         void* stream);

/*
 * Diagnostic: y[i] = 2^x[i] evaluated with the FMA-pipe exponential that the
 * forward kernel uses for part of its softmax terms (range reduction
 * x = rint(x) + f, |f| <= 1/2, then a fitted cubic for 2^f; relative error
 * below 1e-4 for x in [-125, 64]; inputs below -125 give 2^-125). No
 * passage of the FlashAttention pages defines it: the lesson's Researcher
 * section ("Version lineage") names software exponentials on Blackwell, and
 * this entry point lets tests check the one used here against its bound.
 * x and y are device float arrays of n >= 0 elements (NULL allowed when
 * n == 0); asynchronous on `stream`. FA_ERR_INVALID_ARG for n < 0 or NULL
 * pointers with n > 0.
 */
fa_status fa_exp2_fma(const float* x, float* y, long long n, void* stream);

/*
 * Test hook for the bounded-wait contract above ("Errors"); the pages have no
 * counterpart. While on, every launch of the named tensor-core kernels makes
 * its MMA-issuing thread wait first on an mbarrier that nothing ever
 * signals, with a limit of wait_cycles SM clock cycles instead of the normal
 * one of about 1.5 s. That wait runs out, the CTA sets FA_ERR_TIMEOUT's bit
 * in the error word and takes the abort path (its other waits return at once,
 * copies in flight are drained, TMEM is freed) and the kernel returns; CTAs
 * that start after the word is set do nothing. The call's outputs are then
 * undefined; nothing traps, faults or hangs, and after fa_get_device_error
 * has cleared the word the workspace works normally again.
 *   kernels: 0 (off) or an OR of FA_STALL_FWD (fa_fwd tensor-core kernel),
 *            FA_STALL_BWD (backward main kernel), FA_STALL_DQ (the dQ kernel
 *            of fa_bwd_deterministic);
 *   wait_cycles: 1,000 .. 2,000,000,000 when kernels != 0 (ignored when 0).
 * FA_ERR_INVALID_ARG otherwise. Process-wide (every host thread and device),
 * read at each launch; for tests only.
 */
enum { FA_STALL_FWD = 1, FA_STALL_BWD = 2, FA_STALL_DQ = 4 };
fa_status fa_debug_set_stall(int kernels, long long wait_cycles);

/* Number of kernel launches the last successful call of fa_fwd_ex / fa_bwd_ex
 * or one of the stages made from the calling thread (for launch accounting). */
int fa_last_launch_count(void);

/*
 * Reads and clears the workspace's error word: synchronises `stream`, copies
 * the word to the host, then zeroes it. Returns FA_OK if no kernel recorded a
 * failure, FA_ERR_TIMEOUT if a bounded wait ran out, FA_ERR_CUDA if the copy
 * failed (and then leaves the word as it is).
 */
fa_status fa_get_device_error(void* workspace, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
