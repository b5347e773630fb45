// CUDA-core (fp32 FFMA) attention kernels.
//
// These serve the fp32 workload (one head, N = 512, d = 32, the FlashAttention
// lesson's NumPy example), head sizes the tensor-core kernels do not cover,
// and as a second, independent GPU path in the tests. Arithmetic is fp32
// throughout: bf16 inputs are widened on load.
//
// Forward: the online-softmax recurrence of the lesson's Researcher section
// ("Online softmax"): for each key tile j, m_j = max(m_{j-1}, rowmax S_j),
// l_j = e^{m_{j-1}-m_j} l_{j-1} + rowsum e^{S_j - m_j}, O_j likewise, output
// O_T / l_T. Exponentials are taken in base 2 with scale * log2(e) folded into
// the query, so LSE = (m + log2 l) * ln 2.
//
// Backward: P is recomputed from Q, K and the saved LSE (paper summary, "Core
// Idea" item 3). One kernel accumulates dQ over key tiles per query row, a
// second accumulates dK and dV over query tiles (and over the query heads of a
// KV group) per key row; neither uses atomics, so the result is deterministic.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>

#include "internal.h"

namespace fa {
namespace {

namespace cg = cooperative_groups;

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kRows = 32;   // query (or key) rows per CTA
constexpr int kTile = 32;   // keys (or queries) per shared-memory tile
constexpr int kThreads = kRows * 4;  // four threads share one row

template <typename T> __device__ __forceinline__ float ld(const T* p);
template <> __device__ __forceinline__ float ld<float>(const float* p) { return *p; }
template <> __device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ void st(T* p, float v);
template <> __device__ __forceinline__ void st<float>(float* p, float v) { *p = v; }
template <> __device__ __forceinline__ void st<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

// Copies a tile of `kTile` rows x D of a [N, D] matrix into shared memory as
// fp32; rows at or beyond N read as zero.
template <int D, typename T>
__device__ __forceinline__ void load_tile(float (*dst)[D], const T* src, int row0, int N) {
  for (int e = threadIdx.x; e < kTile * D; e += blockDim.x) {
    int r = e / D, c = e % D;
    int gr = row0 + r;
    dst[r][c] = (gr < N) ? ld<T>(src + (size_t)gr * D + c) : 0.f;
  }
}

// ------------------------------------------------------------------ forward

// The online-softmax state of one query row over key tiles j0 = k_begin,
// k_begin + kTile, ... < k_end: running max m (log2 units), sum l and
// unnormalised output o (this thread's D/4 columns: t * 4 + sub).
template <int D, typename T>
__device__ __forceinline__ void fwd_key_range(const Problem& p, float (*Ks)[D], float (*Vs)[D],
                                              const T* Kh, const T* Vh, const float (&q)[D / 4],
                                              int row, int row0, int sub, int k_begin, int k_end,
                                              float& m, float& l, float (&o)[D / 4]) {
  constexpr int DT = D / 4;
  const int N = p.N;
  for (int j0 = k_begin; j0 < k_end; j0 += kTile) {
    if (p.mask && !p.mask[(size_t)(row0 / 128) * p.nb + j0 / 128]) continue;
    __syncthreads();
    load_tile<D, T>(Ks, Kh, j0, N);
    load_tile<D, T>(Vs, Vh, j0, N);
    __syncthreads();
    float s[kTile];
    float mx = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < kTile; ++jj) {
      float a = 0.f;
#pragma unroll
      for (int t = 0; t < DT; ++t) a = fmaf(q[t], Ks[jj][t * 4 + sub], a);
      a = quad_sum(a);
      const int key = j0 + jj;
      if (key >= N || (p.causal && key > row)) a = -INFINITY;
      s[jj] = a;
      mx = fmaxf(mx, a);
    }
    const float m_new = fmaxf(m, mx);
    if (m_new == -INFINITY) continue;  // nothing visible to this row yet
    const float alpha = exp2f(m - m_new);
    l *= alpha;
#pragma unroll
    for (int t = 0; t < DT; ++t) o[t] *= alpha;
#pragma unroll
    for (int jj = 0; jj < kTile; ++jj) {
      const float pj = exp2f(s[jj] - m_new);
      l += pj;
#pragma unroll
      for (int t = 0; t < DT; ++t) o[t] = fmaf(pj, Vs[jj][t * 4 + sub], o[t]);
    }
    m = m_new;
  }
}

template <int D, typename T>
__device__ __forceinline__ void fwd_store_row(const Problem& p, int b, int h, int row, int sub,
                                              float m, float l, const float (&o)[D / 4]) {
  if (row >= p.N) return;
  const size_t base = (((size_t)b * p.Hq + h) * p.N + row);
  T* Oh = static_cast<T*>(p.Oout) + base * D;
  const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
  for (int t = 0; t < D / 4; ++t) st<T>(Oh + t * 4 + sub, o[t] * inv);
  if (sub == 0) p.LSEout[base] = (l > 0.f) ? (m + log2f(l)) * kLn2 : -INFINITY;
}

template <int D, typename T>
__global__ void __launch_bounds__(kThreads) simt_fwd_kernel(Problem p) {
  constexpr int DT = D / 4;
  __shared__ float Ks[kTile][D];
  __shared__ float Vs[kTile][D];
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (p.Hq / p.Hkv);
  const int row0 = blockIdx.x * kRows;
  const int row = row0 + threadIdx.x / 4;
  const int sub = threadIdx.x & 3;
  const int N = p.N;
  const float c = p.scale * kLog2e;
  const T* Qh = static_cast<const T*>(p.Q) + ((size_t)b * p.Hq + h) * N * D;
  const T* Kh = static_cast<const T*>(p.K) + ((size_t)b * p.Hkv + hk) * N * D;
  const T* Vh = static_cast<const T*>(p.V) + ((size_t)b * p.Hkv + hk) * N * D;

  float q[DT], o[DT];
#pragma unroll
  for (int t = 0; t < DT; ++t) {
    q[t] = (row < N) ? ld<T>(Qh + (size_t)row * D + t * 4 + sub) * c : 0.f;
    o[t] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int kend = p.causal ? min(N, row0 + kRows) : N;
  fwd_key_range<D, T>(p, Ks, Vs, Kh, Vh, q, row, row0, sub, 0, kend, m, l, o);
  fwd_store_row<D, T>(p, b, h, row, sub, m, l, o);
}

// The same forward with the key range of each 32-row query block split over
// the CTAs of a thread-block cluster (launched with cluster dimension
// (S, 1, 1), S <= 8): CTA r of the cluster runs the online softmax over its
// share of the key tiles, and rank 0 merges the S partial states (m_r, l_r,
// o_r) row by row through distributed shared memory:
//   m = max_r m_r,  l = sum_r 2^(m_r - m) l_r,  o = sum_r 2^(m_r - m) o_r,
// the same rescaling the recurrence applies tile by tile. Used when a
// problem has too few query blocks to fill the GPU (one head of 512 rows is
// 16 blocks); it needs no global scratch.
template <int D, typename T>
__global__ void __launch_bounds__(kThreads) simt_fwd_split_kernel(Problem p) {
  constexpr int DT = D / 4;
  static_assert(2 * kTile >= kRows, "partial outputs reuse the K and V tiles");
  __shared__ float Ks[kTile][D];
  __shared__ float Vs[kTile][D];
  __shared__ float part_ml[kRows][2];
  cg::cluster_group cl = cg::this_cluster();
  const int S = (int)cl.num_blocks();
  const int split = (int)cl.block_rank();
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (p.Hq / p.Hkv);
  const int row0 = (blockIdx.x / S) * kRows;
  const int r = threadIdx.x / 4;
  const int row = row0 + r;
  const int sub = threadIdx.x & 3;
  const int N = p.N;
  const float c = p.scale * kLog2e;
  const T* Qh = static_cast<const T*>(p.Q) + ((size_t)b * p.Hq + h) * N * D;
  const T* Kh = static_cast<const T*>(p.K) + ((size_t)b * p.Hkv + hk) * N * D;
  const T* Vh = static_cast<const T*>(p.V) + ((size_t)b * p.Hkv + hk) * N * D;

  float q[DT], o[DT];
#pragma unroll
  for (int t = 0; t < DT; ++t) {
    q[t] = (row < N) ? ld<T>(Qh + (size_t)row * D + t * 4 + sub) * c : 0.f;
    o[t] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int kend = p.causal ? min(N, row0 + kRows) : N;
  const int ntile = (kend + kTile - 1) / kTile;
  const int t0 = (int)((long long)split * ntile / S), t1 = (int)((long long)(split + 1) * ntile / S);
  fwd_key_range<D, T>(p, Ks, Vs, Kh, Vh, q, row, row0, sub, t0 * kTile, min(kend, t1 * kTile), m,
                      l, o);
  // partial state into this CTA's shared memory (o over the K/V tiles)
  __syncthreads();
  float* po = &Ks[0][0];   // [kRows][D]
#pragma unroll
  for (int t = 0; t < DT; ++t) po[r * D + t * 4 + sub] = o[t];
  if (sub == 0) {
    part_ml[r][0] = m;
    part_ml[r][1] = l;
  }
  cl.sync();
  if (split == 0) {
    float mm = -INFINITY;
    for (int s = 0; s < S; ++s) mm = fmaxf(mm, cl.map_shared_rank(&part_ml[0][0], s)[2 * r]);
    float ls = 0.f, os[DT];
#pragma unroll
    for (int t = 0; t < DT; ++t) os[t] = 0.f;
    if (mm != -INFINITY) {
      for (int s = 0; s < S; ++s) {
        const float* ml = cl.map_shared_rank(&part_ml[0][0], s);
        const float* ps = cl.map_shared_rank(po, s);
        const float w = exp2f(ml[2 * r] - mm);   // 0 for a split that saw nothing
        ls = fmaf(w, ml[2 * r + 1], ls);
#pragma unroll
        for (int t = 0; t < DT; ++t) os[t] = fmaf(w, ps[r * D + t * 4 + sub], os[t]);
      }
    }
    fwd_store_row<D, T>(p, b, h, row, sub, mm, ls, os);
  }
  cl.sync();   // the other CTAs' shared memory stays alive until rank 0 has read it
}

// ------------------------------------------------------------------ backward

// D_i = sum_k dO_ik O_ik and LSE2_i = LSE_i * log2(e) (+inf for rows with no
// visible key and for padding rows), one warp per row of the padded layout.
// D_i = sum_k dO_ik O_ik and LSE_i * log2(e) for every row of the padded
// [B*Hq][Npad] workspace vectors (padding rows: D = 0, LSE2 = +inf, so their
// P is 0), optionally zeroing the row of the fp32 dQ accumulator. TPR
// threads share a row, each reading 16 bytes of O and of dO (VEC elements),
// and the partial dots are summed with shuffles inside the TPR-lane group.
// Variable-length batches (p.cu set): row r of (b, h) is token cu[b] + r of
// the packed [total][Hq][d] tensors and LSE [Hq][total]; the vectors keep the
// padded [B*Hq][Npad] layout (Npad from the longest sequence).
template <typename T, int TPR>
__global__ void __launch_bounds__(256) preprocess_kernel(Problem p, int zero_acc) {
  constexpr int VEC = 16 / sizeof(T);
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)p.B * p.Hq * p.Npad;
  const long long rowid = gt / TPR;
  const int part = (int)(gt % TPR);
  const bool live = rowid < total;   // whole TPR groups are live or not
  const int bh = live ? (int)(rowid / p.Npad) : 0;
  const int row = live ? (int)(rowid % p.Npad) : p.N;
  const int d = p.d;
  float acc = 0.f;
  int n_rows = p.N;
  size_t row_off = (size_t)bh * p.N + row, lse_off = row_off;   // in units of d / of 1
  if (p.cu && live) {
    const int b = bh / p.Hq, h = bh % p.Hq;
    const int s0 = min(max(p.cu[b], 0), p.total);
    const int s1 = min(max(p.cu[b + 1], s0), p.total);
    n_rows = min(s1 - s0, p.N);
    row_off = (size_t)(s0 + row) * p.Hq + h;
    lse_off = (size_t)h * p.total + s0 + row;
  }
  if (live && row < n_rows) {
    const size_t off = row_off * d + (size_t)part * VEC;
    const uint4 ov = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.O) + off);
    const uint4 gv = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.dO) + off);
    const T* o = reinterpret_cast<const T*>(&ov);
    const T* g = reinterpret_cast<const T*>(&gv);
#pragma unroll
    for (int k = 0; k < VEC; ++k) acc = fmaf(ld<T>(o + k), ld<T>(g + k), acc);
    if (zero_acc) {
      float4* a = reinterpret_cast<float4*>(p.dQacc + off);
#pragma unroll
      for (int k = 0; k < VEC / 4; ++k) a[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (live && part == 0) {
    float lse2 = INFINITY;
    if (row < n_rows) {
      const float L = p.LSE[lse_off];
      if (L != -INFINITY) lse2 = L * kLog2e;
    }
    p.Dws[(size_t)bh * p.Npad + row] = acc;
    p.LSE2ws[(size_t)bh * p.Npad + row] = lse2;
  }
}

template <int D, typename T, typename G>
__global__ void __launch_bounds__(kThreads) simt_dq_kernel(Problem p) {
  constexpr int DT = D / 4;
  __shared__ float Ks[kTile][D];
  __shared__ float Vs[kTile][D];
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (p.Hq / p.Hkv);
  const int row0 = blockIdx.x * kRows;
  const int row = row0 + threadIdx.x / 4;
  const int sub = threadIdx.x & 3;
  const int N = p.N;
  const float c = p.scale * kLog2e;
  const size_t bh = (size_t)b * p.Hq + h;
  const T* Qh = static_cast<const T*>(p.Q) + bh * N * D;
  const T* dOh = static_cast<const T*>(p.dO) + bh * N * D;
  const T* Kh = static_cast<const T*>(p.K) + ((size_t)b * p.Hkv + hk) * N * D;
  const T* Vh = static_cast<const T*>(p.V) + ((size_t)b * p.Hkv + hk) * N * D;
  const int rr = min(row, N - 1);
  const float lse2 = p.LSE2ws[bh * p.Npad + rr];
  const float Di = p.Dws[bh * p.Npad + rr];

  float q[DT], g[DT], dq[DT];
#pragma unroll
  for (int t = 0; t < DT; ++t) {
    q[t] = (row < N) ? ld<T>(Qh + (size_t)row * D + t * 4 + sub) * c : 0.f;
    g[t] = (row < N) ? ld<T>(dOh + (size_t)row * D + t * 4 + sub) : 0.f;
    dq[t] = 0.f;
  }
  const int kend = p.causal ? min(N, row0 + kRows) : N;
  for (int j0 = 0; j0 < kend; j0 += kTile) {
    if (p.mask && !p.mask[(size_t)(row0 / 128) * p.nb + j0 / 128]) continue;
    __syncthreads();
    load_tile<D, T>(Ks, Kh, j0, N);
    load_tile<D, T>(Vs, Vh, j0, N);
    __syncthreads();
#pragma unroll 4
    for (int jj = 0; jj < kTile; ++jj) {
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int t = 0; t < DT; ++t) {
        s = fmaf(q[t], Ks[jj][t * 4 + sub], s);
        dp = fmaf(g[t], Vs[jj][t * 4 + sub], dp);
      }
      s = quad_sum(s);
      dp = quad_sum(dp);
      const int key = j0 + jj;
      const bool vis = row < N && key < N && !(p.causal && key > row);
      const float pj = vis ? exp2f(s - lse2) : 0.f;
      const float ds = pj * (dp - Di);
#pragma unroll
      for (int t = 0; t < DT; ++t) dq[t] = fmaf(ds, Ks[jj][t * 4 + sub], dq[t]);
    }
  }
  if (row < N) {
    G* out = static_cast<G*>(p.dQ) + (bh * N + row) * D;
#pragma unroll
    for (int t = 0; t < DT; ++t) st<G>(out + t * 4 + sub, dq[t] * p.scale);
  }
}

template <int D, typename T, typename G>
__global__ void __launch_bounds__(kThreads) simt_dkdv_kernel(Problem p) {
  constexpr int DT = D / 4;
  __shared__ float Qs[kTile][D];
  __shared__ float Gs[kTile][D];
  __shared__ float Ls[kTile];
  __shared__ float Ds[kTile];
  const int hk = blockIdx.y, b = blockIdx.z;
  const int grp = p.Hq / p.Hkv;
  const int key0 = blockIdx.x * kRows;
  const int key = key0 + threadIdx.x / 4;
  const int sub = threadIdx.x & 3;
  const int N = p.N;
  const float c = p.scale * kLog2e;
  const size_t bk = (size_t)b * p.Hkv + hk;
  const T* Kh = static_cast<const T*>(p.K) + bk * N * D;
  const T* Vh = static_cast<const T*>(p.V) + bk * N * D;

  float k[DT], v[DT], dk[DT], dv[DT];
#pragma unroll
  for (int t = 0; t < DT; ++t) {
    k[t] = (key < N) ? ld<T>(Kh + (size_t)key * D + t * 4 + sub) * c : 0.f;
    v[t] = (key < N) ? ld<T>(Vh + (size_t)key * D + t * 4 + sub) : 0.f;
    dk[t] = 0.f;
    dv[t] = 0.f;
  }
  const int istart = p.causal ? key0 : 0;
  for (int hh = 0; hh < grp; ++hh) {
    const size_t bh = (size_t)b * p.Hq + hk * grp + hh;
    const T* Qh = static_cast<const T*>(p.Q) + bh * N * D;
    const T* dOh = static_cast<const T*>(p.dO) + bh * N * D;
    for (int i0 = istart; i0 < N; i0 += kTile) {
      if (p.mask && !p.mask[(size_t)(i0 / 128) * p.nb + key0 / 128]) continue;
      __syncthreads();
      load_tile<D, T>(Qs, Qh, i0, N);
      load_tile<D, T>(Gs, dOh, i0, N);
      if (threadIdx.x < kTile) {
        const int r = i0 + threadIdx.x;
        Ls[threadIdx.x] = (r < N) ? p.LSE2ws[bh * p.Npad + r] : INFINITY;
        Ds[threadIdx.x] = (r < N) ? p.Dws[bh * p.Npad + r] : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int ii = 0; ii < kTile; ++ii) {
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int t = 0; t < DT; ++t) {
          s = fmaf(k[t], Qs[ii][t * 4 + sub], s);
          dp = fmaf(v[t], Gs[ii][t * 4 + sub], dp);
        }
        s = quad_sum(s);
        dp = quad_sum(dp);
        const int qi = i0 + ii;
        const bool vis = key < N && qi < N && !(p.causal && key > qi);
        const float pj = vis ? exp2f(s - Ls[ii]) : 0.f;
        const float ds = pj * (dp - Ds[ii]);
#pragma unroll
        for (int t = 0; t < DT; ++t) {
          dv[t] = fmaf(pj, Gs[ii][t * 4 + sub], dv[t]);
          dk[t] = fmaf(ds, Qs[ii][t * 4 + sub], dk[t]);
        }
      }
    }
  }
  if (key < N) {
    G* ok = static_cast<G*>(p.dK) + (bk * N + key) * D;
    G* ov = static_cast<G*>(p.dV) + (bk * N + key) * D;
#pragma unroll
    for (int t = 0; t < DT; ++t) {
      st<G>(ok + t * 4 + sub, dk[t] * p.scale);
      st<G>(ov + t * 4 + sub, dv[t]);
    }
  }
}

template <typename G>
__global__ void __launch_bounds__(256) dq_convert_kernel(const float* __restrict__ acc,
                                                        G* __restrict__ out, size_t n4) {
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (; i < n4; i += stride) {
    const float4 v = reinterpret_cast<const float4*>(acc)[i];
    G* o = out + i * 4;
    st<G>(o + 0, v.x);
    st<G>(o + 1, v.y);
    st<G>(o + 2, v.z);
    st<G>(o + 3, v.w);
  }
}

// ------------------------------------------------------------------ dispatch

template <int D, typename T>
cudaError_t launch_fwd(const Problem& p) {
  const long long nblk = (p.N + kRows - 1) / kRows;
  const long long blocks = nblk * p.Hq * p.B;
  // Too few query blocks to fill the 148 SMs: split each block's key tiles
  // over a cluster of S CTAs (S a power of two, at most 8 and at most the
  // block's key tiles), merged through distributed shared memory.
  int S = 1;
  const long long ktiles = (p.N + kTile - 1) / kTile;
  while (S < 8 && blocks * S < 148 && 2 * S <= ktiles) S *= 2;
  if (S == 1) {
    dim3 grid((unsigned)nblk, p.Hq, p.B);
    simt_fwd_kernel<D, T><<<grid, kThreads, 0, p.stream>>>(p);
  } else {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(nblk * S), p.Hq, p.B);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = p.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, simt_fwd_split_kernel<D, T>, p);
    if (e != cudaSuccess) return e;
  }
  count_launch();
  return cudaGetLastError();
}

template <int D, typename T, typename G>
cudaError_t launch_bwd(const Problem& p) {
  dim3 g1((p.N + kRows - 1) / kRows, p.Hq, p.B);
  simt_dq_kernel<D, T, G><<<g1, kThreads, 0, p.stream>>>(p);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2((p.N + kRows - 1) / kRows, p.Hkv, p.B);
  simt_dkdv_kernel<D, T, G><<<g2, kThreads, 0, p.stream>>>(p);
  count_launch();
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_bwd_d(const Problem& p) {
  if (p.dtype == 0) {
    return p.grad_dtype == 0 ? launch_bwd<D, float, float>(p)
                             : launch_bwd<D, float, __nv_bfloat16>(p);
  }
  return p.grad_dtype == 0 ? launch_bwd<D, __nv_bfloat16, float>(p)
                           : launch_bwd<D, __nv_bfloat16, __nv_bfloat16>(p);
}

}  // namespace

cudaError_t simt_fwd(const Problem& p) {
  const bool f32 = p.dtype == 0;
  switch (p.d) {
    case 16: return f32 ? launch_fwd<16, float>(p) : launch_fwd<16, __nv_bfloat16>(p);
    case 32: return f32 ? launch_fwd<32, float>(p) : launch_fwd<32, __nv_bfloat16>(p);
    case 64: return f32 ? launch_fwd<64, float>(p) : launch_fwd<64, __nv_bfloat16>(p);
    case 128: return f32 ? launch_fwd<128, float>(p) : launch_fwd<128, __nv_bfloat16>(p);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, int TPR>
cudaError_t launch_preprocess(const Problem& p, bool zero_acc) {
  const long long threads = (long long)p.B * p.Hq * p.Npad * TPR;
  const long long blocks = (threads + 255) / 256;
  preprocess_kernel<T, TPR><<<(unsigned)blocks, 256, 0, p.stream>>>(p, zero_acc ? 1 : 0);
  count_launch();
  return cudaGetLastError();
}

template <typename T>
cudaError_t preprocess_d(const Problem& p, bool zero_acc) {
  constexpr int VEC = 16 / sizeof(T);
  switch (p.d / VEC) {
    case 2: return launch_preprocess<T, 2>(p, zero_acc);
    case 4: return launch_preprocess<T, 4>(p, zero_acc);
    case 8: return launch_preprocess<T, 8>(p, zero_acc);
    case 16: return launch_preprocess<T, 16>(p, zero_acc);
    case 32: return launch_preprocess<T, 32>(p, zero_acc);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t bwd_preprocess(const Problem& p, bool zero_acc) {
  return p.dtype == 0 ? preprocess_d<float>(p, zero_acc) : preprocess_d<__nv_bfloat16>(p, zero_acc);
}

cudaError_t simt_bwd_main(const Problem& p) {
  switch (p.d) {
    case 16: return launch_bwd_d<16>(p);
    case 32: return launch_bwd_d<32>(p);
    case 64: return launch_bwd_d<64>(p);
    case 128: return launch_bwd_d<128>(p);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t dq_convert(const Problem& p) {
  const size_t rows = p.cu ? (size_t)p.total : (size_t)p.B * p.N;
  const size_t n = rows * p.Hq * p.d;  // d is a multiple of 16
  const size_t n4 = n / 4;
  if (n4 == 0) return cudaSuccess;
  const int blocks = (int)std::min<size_t>((n4 + 255) / 256, 148 * 16);
  if (p.grad_dtype == 0)
    dq_convert_kernel<float><<<blocks, 256, 0, p.stream>>>(p.dQacc, static_cast<float*>(p.dQ), n4);
  else
    dq_convert_kernel<__nv_bfloat16><<<blocks, 256, 0, p.stream>>>(
        p.dQacc, static_cast<__nv_bfloat16*>(p.dQ), n4);
  count_launch();
  return cudaGetLastError();
}

}  // namespace fa
