// sm_100a building blocks written as inline PTX: mbarriers with bounded waits,
// TMA tensor copies, tcgen05 tensor-memory allocation, MMA, loads and stores,
// and the shared-memory / instruction descriptors the MMAs take.
//
// Descriptor formats follow the PTX ISA description of tcgen05 (matrix
// descriptor: start address, leading / stride byte offsets, version 1,
// swizzle mode; instruction descriptor for kind::f16: D format, A/B formats,
// major-ness, N >> 3, M >> 4).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace fa {
namespace sm100 {

// ---------------------------------------------------------------- misc

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool elect_lane0() { return (threadIdx.x & 31) == 0; }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Two-lane fp32 FMA / add / multiply (fma.rn.f32x2 and friends).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

// 2^x for two lanes on the FMA pipe instead of the MUFU unit. Cody and
// Waite's range reduction in base 2 splits x = j + f with j = rint(x) and
// |f| <= 1/2 (adding 1.5 * 2^23 leaves rint(x) in the low mantissa bits of
// the sum); 2^f is a cubic whose coefficients are the relative-error
// least-squares fit printed by exp2_poly_fit.py (max relative error 7.7e-5),
// and 2^j is added to the exponent field. Inputs below -125 are clamped to
// -125 so the exponent stays normal: the result is then 2^-125 instead of a
// smaller number. Not for -inf (masked scores): callers use ex2() there.
constexpr float kExp2P0 = 9.999289513e-01f, kExp2P1 = 6.932762265e-01f,
                kExp2P2 = 2.426040471e-01f, kExp2P3 = 5.508868396e-02f;
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kRound = 12582912.0f;   // 1.5 * 2^23
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 t = fadd2(x, make_float2(kRound, kRound));
  const float2 j = fadd2(t, make_float2(-kRound, -kRound));
  const float2 f = ffma2(j, make_float2(-1.0f, -1.0f), x);
  float2 q = ffma2(make_float2(kExp2P3, kExp2P3), f, make_float2(kExp2P2, kExp2P2));
  q = ffma2(q, f, make_float2(kExp2P1, kExp2P1));
  q = ffma2(q, f, make_float2(kExp2P0, kExp2P0));
  return make_float2(__int_as_float(__float_as_int(q.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(q.y) + (__float_as_int(t.y) << 23)));
}

// tanh(u) = 1 - 2 / (1 + e^(2u)) from the MUFU base-2 exponential and a fast
// reciprocal; absolute error about 1e-7 (u is clamped to [-20, 20], where
// tanh is +-1 to float precision, so the exponential stays finite). Used by
// the soft-capping score modifier.
__device__ __forceinline__ float tanh_ex2(float u) {
  u = fminf(fmaxf(u, -20.f), 20.f);
  const float e = ex2(u * 2.8853900817779268f);   // 2 log2(e)
  return 1.f - __fdividef(2.f, 1.f + e);
}

// Named barrier among `count` threads (a multiple of 32).
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ---------------------------------------------------------------- bounded waits

// Wait limit in SM clock cycles (about one to two seconds): far above any
// legitimate wait of these kernels, short enough that a broken pipeline ends
// with an error word instead of a hung GPU.
constexpr long long kWaitLimitCycles = 3000000000ll;

// Shared abort flag plus the device error word. Once any thread's wait runs
// out, every later wait in the CTA returns at once (false), so all roles run
// their loops to the end without blocking and the CTA exits normally.
struct Guard {
  volatile int* abort;
  unsigned* err;
};

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete. Returns false if the
// CTA has aborted or the wait ran out (which then aborts the CTA). `limit` is
// the wait limit in SM clock cycles.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const Guard& g,
                                          long long limit = kWaitLimitCycles) {
  if (*g.abort) return false;
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*g.abort) return false;
    if (clock64() - t0 > limit) {
      *g.abort = 1;
      atomicOr(g.err, kErrTimeout);
      __threadfence();
      return false;
    }
  }
}

// mbar_wait with the checks in the other order: a phase that has already
// completed is taken before the abort flag is read, so the fast path is one
// shared-memory operation instead of two. Used where the waits sit on the
// MMA issue chain (the forward kernels: measured 5-7 % faster on B200; the
// backward main kernel measured 1 % slower with it and keeps mbar_wait).
__device__ __forceinline__ bool mbar_wait_ready_first(uint64_t* bar, uint32_t parity,
                                                      const Guard& g,
                                                      long long limit = kWaitLimitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait(bar, parity, g, limit);
}

// Test hook of the bounded-wait contract: when stall_cycles > 0 the caller
// waits on `never`, a barrier initialised with one expected arrival that
// nothing ever signals, with that short limit. The wait runs out and takes
// the normal abort path (error word set, every other wait of the CTA returns
// at once, in-flight copies and MMAs are drained, TMEM is freed). Returns
// false after such a stall; true (without waiting) when stall_cycles <= 0.
__device__ __forceinline__ bool injected_stall(uint64_t* never, long long stall_cycles,
                                               const Guard& g) {
  if (stall_cycles <= 0) return true;
  return mbar_wait(never, 0, g, stall_cycles);
}

// ---------------------------------------------------------------- mask modifiers

// Which keys a query sees, before the 128 x 128 block mask (a mask modifier
// in the FlexAttention sense: one tiled kernel, many masks). Key j is visible
// to query i iff lo(i) <= j <= hi(i), where
//   hi(i) = min(wr >= 0 ? max(i + wr, prefix - 1) : N - 1, last row of i's document)
//   lo(i) = max(wl >= 0 ? i - wl : 0, first row of i's document)
// The causal flag is the window wr = 0; prefix > 0 makes the first `prefix`
// keys visible to every query whatever the right bound says (prefix LM);
// doc lists one document id per token, non-decreasing, and a query sees only
// its own document. lo and hi are non-decreasing in i, so the queries that see
// key j form an interval too, and the visibility of a tile follows from its
// corner rows and columns.
struct MaskMod {
  int wl, wr;          // window bounds, -1 unbounded (the causal flag sets wr = 0)
  int prefix;          // keys below this are visible to every query (0: none)
  const int* doc;      // [N] non-decreasing document ids, or null
};

// First and last row of the run of equal ids that contains row i (binary
// searches over [0, i] and [i, N - 1]). Ids that are not sorted give wrong
// runs but no access outside doc[0 .. N-1].
__device__ __forceinline__ int doc_first(const int* doc, int i) {
  const int t = doc[i];
  int a = 0, b = i;
  while (a < b) {
    const int mid = (a + b) >> 1;
    if (doc[mid] < t) a = mid + 1; else b = mid;
  }
  return a;
}
__device__ __forceinline__ int doc_last(const int* doc, int i, int N) {
  const int t = doc[i];
  int a = i, b = N - 1;
  while (a < b) {
    const int mid = (a + b + 1) >> 1;
    if (doc[mid] > t) b = mid - 1; else a = mid;
  }
  return a;
}

// Keys [lo, hi] that query row i sees (empty when lo > hi). Rows at or past N
// get the interval of row N - 1 (their results are never stored).
__device__ __forceinline__ void mod_row_keys(const MaskMod& m, int i, int N, int& lo, int& hi) {
  hi = N - 1;
  lo = 0;
  if (m.wr >= 0) hi = min(hi, max(i + m.wr, m.prefix - 1));
  if (m.wl >= 0) lo = max(0, i - m.wl);
  if (m.doc) {
    const int r = min(i, N - 1);
    lo = max(lo, doc_first(m.doc, r));
    hi = min(hi, doc_last(m.doc, r, N));
  }
}

// Queries [qlo, qhi] that see key j (empty when qlo > qhi; keys at or past N
// see nothing).
__device__ __forceinline__ void mod_key_queries(const MaskMod& m, int j, int N, int& qlo,
                                                int& qhi) {
  qlo = 0;
  qhi = N - 1;
  if (j >= N) {
    qhi = -1;
    return;
  }
  if (m.wr >= 0 && j >= m.prefix) qlo = max(0, j - m.wr);
  if (m.wl >= 0) qhi = min(qhi, j + m.wl);
  if (m.doc) {
    qlo = max(qlo, doc_first(m.doc, j));
    qhi = min(qhi, doc_last(m.doc, j, N));
  }
}

enum : int { kTileEmpty = 0, kTilePartial = 1, kTileFull = 2 };

// Visibility of the tile of query rows [r0, r1] and keys [c0, c1] (r0, c0 <
// N) under the modifier, before the block mask: kTileEmpty if no pair is
// visible, kTileFull if every pair is (and the tile lies inside the
// sequence), kTilePartial otherwise. Exact for the window and the prefix;
// with documents a tile may be called partial although it is empty (its
// elements are then all masked), never the reverse.
__device__ __forceinline__ int mod_classify(const MaskMod& m, int r0, int r1, int c0, int c1,
                                            int N) {
  const int hi_max = (m.wr >= 0) ? max(r1 + m.wr, m.prefix - 1) : 0x7fffffff;
  const int lo_min = (m.wl >= 0) ? r0 - m.wl : -0x7fffffff;
  if (c0 > hi_max || c1 < lo_min) return kTileEmpty;
  const int hi_min = (m.wr >= 0) ? max(r0 + m.wr, m.prefix - 1) : 0x7fffffff;
  const int lo_max = (m.wl >= 0) ? r1 - m.wl : -0x7fffffff;
  bool full = c1 <= hi_min && c0 >= lo_max && r1 < N && c1 < N;
  if (m.doc) {
    const int dr0 = m.doc[r0], dr1 = m.doc[min(r1, N - 1)];
    const int dc0 = m.doc[c0], dc1 = m.doc[min(c1, N - 1)];
    if (dc1 < dr0 || dc0 > dr1) return kTileEmpty;   // no document in common
    full = full && dr0 == dr1 && dc0 == dc1 && dr0 == dc0;
  }
  return full ? kTileFull : kTilePartial;
}

// Last key any of the query rows [r0, r1] can see, before documents: the
// key-tile range of a query block ends there.
__device__ __forceinline__ int mod_last_key(const MaskMod& m, int r1, int N) {
  return (m.wr >= 0) ? min(N - 1, max(r1 + m.wr, m.prefix - 1)) : N - 1;
}

// First query that can see any of the keys [c0, ...], before documents.
__device__ __forceinline__ int mod_first_query(const MaskMod& m, int c0) {
  return (m.wr >= 0 && c0 >= m.prefix) ? max(0, c0 - m.wr) : 0;
}

// Maps a linear CTA index to (head, block) so that the blocks of `chunk`
// heads are interleaved and, inside the chunk, issued from block 0 to
// block nblk-1 (callers order their blocks by decreasing work). A wave then
// covers only a few heads (their K/V or Q/dO stay in L2) while the longest
// blocks of each chunk start first.
__device__ __forceinline__ void chunked_order(int lin, int nblk, int BH, int chunk, int& head,
                                              int& blk) {
  const int per = chunk * nblk;
  const int c = lin / per, rem = lin - c * per;
  const int heads = min(chunk, BH - c * chunk);
  blk = rem / heads;
  head = c * chunk + (rem - blk * heads);
}

// ---------------------------------------------------------------- TMA

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 3-D tiled load of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Plain (untiled) bulk copy global -> shared; addresses and size 16-byte multiples.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 3-D tiled reduce-add of a shared-memory box into global memory (fp32 add).
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* m, const void* src, int x,
                                                  int y, int z) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group"
      " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(m)),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// 3-D tiled store of a shared-memory box into global memory.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* m, const void* src, int x, int y,
                                             int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group"
      " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(m)),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Makes generic-proxy shared-memory writes visible to the async proxy (TMA / MMA).
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tensor memory

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// TMEM address of (lane, column).
__device__ __forceinline__ uint32_t taddr(uint32_t base, uint32_t lane, uint32_t col) {
  return base + (lane << 16) + col;
}

#define FA_R8(i) "=r"(r[i + 0]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
                 "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define FA_W8(i) "r"(r[i + 0]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), \
                 "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// 32 consecutive 32-bit columns of this thread's lane, waited for before return.
__device__ __forceinline__ void tmem_ld32(uint32_t ta, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : FA_R8(0), FA_R8(8), FA_R8(16), FA_R8(24)
      : "r"(ta)
      : "memory");
}

// 64 consecutive columns (two loads, one wait).
__device__ __forceinline__ void tmem_ld64(uint32_t ta, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : FA_R8(0), FA_R8(8), FA_R8(16), FA_R8(24), FA_R8(32), FA_R8(40), FA_R8(48), FA_R8(56)
      : "r"(ta), "r"(ta + 32)
      : "memory");
}

// 128 consecutive columns (four loads, one wait).
__device__ __forceinline__ void tmem_ld128(uint32_t ta, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%128];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%129];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,"
      "%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95}, [%130];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,"
      "%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%131];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : FA_R8(0), FA_R8(8), FA_R8(16), FA_R8(24), FA_R8(32), FA_R8(40), FA_R8(48), FA_R8(56),
        FA_R8(64), FA_R8(72), FA_R8(80), FA_R8(88), FA_R8(96), FA_R8(104), FA_R8(112),
        FA_R8(120)
      : "r"(ta), "r"(ta + 32), "r"(ta + 64), "r"(ta + 96)
      : "memory");
}

// 32 consecutive columns stored from registers (not waited for).
__device__ __forceinline__ void tmem_st32(uint32_t ta, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(ta),
      FA_W8(0), FA_W8(8), FA_W8(16), FA_W8(24)
      : "memory");
}

#define FA_W4(i) "r"(r[i + 0]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3])

// 16 consecutive 32-bit columns stored from registers (not waited for).
__device__ __forceinline__ void tmem_st16(uint32_t ta, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(ta),
      FA_W8(0), FA_W8(8)
      : "memory");
}

// Two loads of 32 columns each (from two addresses), one wait.
__device__ __forceinline__ void tmem_ld32x2(uint32_t ta, uint32_t tb, uint32_t (&a)[32],
                                            uint32_t (&b)[32]) {
  uint32_t(&r)[32] = a;
  uint32_t(&q)[32] = b;
#define FA_Q8(i) "=r"(q[i + 0]), "=r"(q[i + 1]), "=r"(q[i + 2]), "=r"(q[i + 3]), \
                 "=r"(q[i + 4]), "=r"(q[i + 5]), "=r"(q[i + 6]), "=r"(q[i + 7])
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : FA_R8(0), FA_R8(8), FA_R8(16), FA_R8(24), FA_Q8(0), FA_Q8(8), FA_Q8(16), FA_Q8(24)
      : "r"(ta), "r"(tb)
      : "memory");
#undef FA_Q8
}

// 32 consecutive columns, asynchronous: the registers are valid only after
// tmem_wait_ld(r) on the same array (which also orders their later uses).
__device__ __forceinline__ void tmem_ld32_async(uint32_t ta, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : FA_R8(0), FA_R8(8), FA_R8(16), FA_R8(24)
      : "r"(ta)
      : "memory");
}

#define FA_RW8(i) "+r"(r[i + 0]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), \
                  "+r"(r[i + 4]), "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7])
// Waits for this thread's outstanding TMEM loads; `r` is passed through so the
// compiler cannot move uses of the loaded registers above the wait.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : FA_RW8(0), FA_RW8(8), FA_RW8(16), FA_RW8(24)
               :
               : "memory");
}
#undef FA_RW8

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- MMA

// Shared-memory matrix descriptor, 128-byte swizzle. Addresses in bytes.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version for sm_100
  d |= static_cast<uint64_t>(2) << 61;  // SWIZZLE_128B
  return d;
}

// Descriptor of the operand `off` bytes (a multiple of 16) past the one `d`
// describes, with the same layout: the start-address field holds the address
// / 16 in its low 14 bits and shared memory ends below 256 KB, so adding
// off / 16 never carries out of the field. Cheaper than rebuilding the
// descriptor on an MMA issue path.
__device__ __forceinline__ uint64_t sdesc_at(uint64_t d, uint32_t off) { return d + (off >> 4); }

// Instruction descriptor, kind::f16: bf16 x bf16 -> f32, dense.
// a_mn / b_mn: operand is MN-major (else K-major).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4)                                  // D format f32
         | (1u << 7)                                // A format bf16
         | (1u << 10)                               // B format bf16
         | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// D(tmem) (+)= A(smem) * B(smem)
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// D(tmem) (+)= A(tmem) * B(smem)
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                       uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// Arrives once on `bar` when all previously issued MMAs of this thread are done.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

}  // namespace sm100

// ---------------------------------------------------------------- host side

// Builds a 3-D tiled tensor map over a [planes][rows][cols] row-major tensor
// (cols contiguous). Box = {box_cols, box_rows, 1}. Returns false on failure.
bool make_tmap_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
                  uint64_t cols, uint64_t rows, uint64_t planes, uint32_t box_cols,
                  uint32_t box_rows, CUtensorMapSwizzle swz);
// As make_tmap_3d with explicit row and plane strides (in elements), e.g. the
// packed [total][H][d] layout of variable-length batches: rows = tokens
// (stride H*d), planes = heads (stride d).
bool make_tmap_3d_strided(CUtensorMap* m, const void* base, CUtensorMapDataType dt,
                          int elem_bytes, uint64_t cols, uint64_t rows, uint64_t planes,
                          uint64_t row_stride, uint64_t plane_stride, uint32_t box_cols,
                          uint32_t box_rows, CUtensorMapSwizzle swz);
// Sets cudaFuncAttributeMaxDynamicSharedMemorySize of kernel `fn` to `bytes`
// on the current device, once per (device, kernel, size); thread-safe.
cudaError_t set_max_dynamic_smem(const void* fn, int bytes);
// The kernels' mask modifier for a problem: the causal flag becomes the right
// window bound 0 (it wins over a wider one); a bound of N or more cuts
// nothing and becomes unbounded (which keeps row +- bound inside int range).
inline sm100::MaskMod mask_mod_of(const Problem& p) {
  sm100::MaskMod m;
  m.wl = (p.wl >= p.N) ? -1 : p.wl;
  m.wr = p.causal ? 0 : ((p.wr >= p.N) ? -1 : p.wr);
  m.prefix = (p.prefix > p.N) ? p.N : p.prefix;
  m.doc = p.doc;
  return m;
}
// The map of a [B][H][N][cols] tensor (dense) or of a packed [total][H][cols]
// one (variable-length, p.cu set); rows of the box run over N or tokens.
inline bool make_seq_tmap(CUtensorMap* m, const Problem& p, const void* base,
                          CUtensorMapDataType dt, int elem_bytes, int H, uint32_t box_cols,
                          uint32_t box_rows, CUtensorMapSwizzle swz) {
  const uint64_t d = (uint64_t)p.d;
  if (p.cu)
    return make_tmap_3d_strided(m, base, dt, elem_bytes, d, (uint64_t)p.total, (uint64_t)H,
                                (uint64_t)H * d, d, box_cols, box_rows, swz);
  return make_tmap_3d(m, base, dt, elem_bytes, d, (uint64_t)p.N, (uint64_t)p.B * H, box_cols,
                      box_rows, swz);
}

}  // namespace fa
