// Attention backward for sm_100a: one CTA per 128-key tile of one (batch, KV
// head), tcgen05 MMAs with dK and dV accumulated in TMEM for the whole CTA,
// P recomputed on chip from Q, K and the forward's LSE (paper summary, "Core
// Idea" item 3: recomputation instead of storing the N x N matrix).
//
// For each visible (query head of the KV group, query tile) item i:
//
//   S^T  = K Q_i^T                 SS MMA -> TMEM
//   dP^T = V dO_i^T                SS MMA -> TMEM
//   P^T  = exp2(S^T * scale*log2e - LSE2_i)      softmax warps, one key row per thread
//   dS^T = P^T * (dP^T - D_i)                    (D_i = rowsum(dO_i * O_i), preprocess)
//   dV  += P^T dO_i                TS MMA (P^T bf16 in TMEM)
//   dK  += dS^T Q_i                SS MMA (dS^T bf16 in shared memory)
//   dQ_i = dS_i K   (d = 64)  or  dQ_i^T = K^T dS_i^T   (d = 128)   SS MMA -> TMEM
//   dQ accumulator += scale * dQ_i  TMA reduce-add from shared memory
//
// Query tiles are 128 rows for d = 64 and 64 rows for d = 128 so that every
// accumulator fits the 512 TMEM columns; the dQ product is arranged so its
// M dimension is 128 either way.
//
// Schedule (d = 128): two sets of S^T / dP^T columns in TMEM alternate
// between items, so the softmax of item i+1 runs while the tensor core does
// dV(i), dK(i), dQ(i). MMA issue order for item i: dV(i), dK(i), dQ(i) (into
// the S columns of its own set, which dV(i) has finished reading: tcgen05.mma
// operations issued by one thread run in order), then dP(i+2) and, once the
// drain warps have read dQ(i), S(i+2) into the same set. Q / dO use a
// three-stage ring.
// Schedule (d = 64, where two sets do not fit): one set; order dV(i),
// S(i+1), dP(i+1), dK(i), dQ(i) into its own columns.
// In both, the dS^T shared buffer alternates by item parity and the softmax
// of item i only writes it after the MMAs that read it two items earlier
// have completed (they precede the S MMA it waited for).
//
// Warp roles: warp 0 TMA producer, warp 1 MMA issuer, warp 2 TMEM
// allocator, warp 3 builds the query-tile list, then the softmax / dS warps
// (which also store dK and dV at the end): 4 for d = 128, 8 for d = 64 (two
// per TMEM lane quarter, each on half of the item's query columns), then 4
// warps that drain dQ from TMEM to the global fp32 accumulator. P^T of each
// 32-column chunk goes to the first 16 of that chunk's own S columns, so
// warps on different chunks never touch each other's scores.
#include <math.h>

#include <algorithm>

#include "sm100_common.cuh"

namespace fa {
namespace {
using namespace sm100;

constexpr int kBN = 128;            // keys per CTA
constexpr int kMaxQTiles = 4096;    // query tiles per sequence
// KV heads interleaved in launch order (build-time tuning; default measured
// on B200)
#ifndef FA_BWD_CHUNK
#define FA_BWD_CHUNK 8
#endif
constexpr int kChunk = FA_BWD_CHUNK;
// 1: at d = 128 the two softmax warpgroups take alternate items (build-time
// choice for A/B measurements; 0: one warpgroup takes every item).
#ifndef FA_BWD_ITEM_SPLIT
#define FA_BWD_ITEM_SPLIT 0
#endif
// d = 128, dense batches: 1 lets the dQ drain warps stage and store dV while
// the softmax warps do dK (0: the softmax warps do both, one after the other).
#ifndef FA_BWD_DV_DRAIN
#define FA_BWD_DV_DRAIN 1
#endif
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
  // Softmax / dS warps, in groups of four (one warp per TMEM lane quarter).
  // d = 64: two groups, each on half of every item's query columns (measured
  // 17% faster on B200 than one group). d = 128: two groups taking alternate
  // items, each on its own S^T / dP^T set in TMEM, dS^T buffer and p_ready
  // barrier, so the softmax of two items runs at once (one group on every
  // item left the MMA warp waiting: the per-item softmax / dS step is
  // latency-bound at one warp per SMSP).
  static constexpr bool kItemSplit = (D == 128) && FA_BWD_ITEM_SPLIT;
  static constexpr int kSoftWarps = (D == 64 || kItemSplit) ? 8 : 4;
  static constexpr int kColHalves = (D == 64) ? 2 : 1;    // groups sharing an item's columns
  static constexpr int kThreads = (8 + kSoftWarps) * 32;
  static constexpr bool kDrainDV = kSoftWarps == 4 && FA_BWD_DV_DRAIN;
  static constexpr bool kDbl = (D == 128);                // two S/dP sets in TMEM
  static constexpr int MQ = (D == 64) ? 128 : 64;         // query rows per item
  static constexpr int kStages = kDbl ? 3 : 2;            // Q / dO ring depth
  static constexpr int kKVBytes = kBN * D * 2;            // K or V tile
  static constexpr int kQBytes = MQ * D * 2;              // Q or dO tile
  static constexpr int kQBlock = MQ * 128;                // one 64-column block of Q / dO
  static constexpr int kDSBytes = kBN * MQ * 2;           // dS^T buffer (bf16)
  static constexpr int kStgBox = MQ * 128;                // one 32-column fp32 box of dQ
  static constexpr int kStgBoxes = kDbl ? 2 : D / 32;     // boxes staged at a time
  // TMEM columns
  static constexpr uint32_t kDK = 0, kDV = D;
  static constexpr uint32_t kS0 = 2 * D, kDP0 = 2 * D + MQ;
  static constexpr uint32_t kS1 = kDbl ? 2 * D + 2 * MQ : kS0;
  static constexpr uint32_t kDP1 = kDbl ? 2 * D + 3 * MQ : kDP0;
  static constexpr uint32_t kDQ = 2 * D + 2 * MQ;         // dQ columns of the one-set schedule
  // shared memory (offsets from a 1024-aligned base)
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKVBytes;
  static constexpr int kOffQ = kOffV + kKVBytes;
  static constexpr int kOffDO = kOffQ + kStages * kQBytes;
  static constexpr int kOffDS = kOffDO + kStages * kQBytes;
  static constexpr int kOffStg = kOffDS + 2 * kDSBytes;
  static constexpr int kOffVec = kOffStg + kStgBoxes * kStgBox;   // [stage][LSE2 | D][MQ]
  static constexpr int kOffEnd = kOffVec + kStages * 2 * MQ * 4;
  static_assert((kDbl ? kDP1 + MQ : kDQ + 64) <= 512, "TMEM budget");
  // the dK / dV epilogue stages both fp32 tensors over the Q/dO ring and the
  // dS buffers, which lie back to back before the dQ staging
  static_assert(kOffStg - kOffQ >= 2 * kBN * D * 4, "epilogue staging");
};

struct alignas(16) Ctl {
  uint64_t kv_full;
  uint64_t qdo_full[3], qdo_empty[3];
  uint64_t sp_full[2], p_ready[2], dq_full, dq_free, acc_done;
  uint64_t never;              // signalled by nothing (wait-limit test hook)
  uint32_t tmem_base;
  int abort;
  int skip;                    // the error word was set at launch: the CTA does nothing
  int nq;                      // visible query tiles per query head
  uint16_t qtiles[kMaxQTiles];  // visible query tiles, | kFullBit
};

// Flag on a query-tile entry: every (query, key) pair of the item is
// visible, so its scores need no masking.
constexpr uint16_t kFullBit = 0x8000;

// Stages one thread's row r of a 128 x D gradient accumulator (TMEM columns
// from taddr; zeros when the CTA ran no item) at st, in the TMA's
// 128-byte-swizzled layout: box b (128 bytes of each row: 32 fp32 or 64 bf16
// columns) at b * 16 KB, row r at r * 128 bytes, 16-byte chunk c at
// ((c ^ (r & 7)) << 4).
template <int D>
__device__ __forceinline__ void stage_grad(uint8_t* st, uint32_t taddr, bool have, float mul,
                                           bool grad_bf16, int r) {
#pragma unroll 1
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t v[32];
    if (have) {
      tmem_ld32(taddr + cc * 32, v);
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = 0u;
    }
    if (grad_bf16) {
      // 32 columns = 64 bytes: chunks 4 (cc & 1) .. +3 of box cc / 2
      uint32_t w[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        w[e] = pack_bf16(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
      uint8_t* rowp = st + (cc >> 1) * 16384 + r * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int c = 4 * (cc & 1) + q;
        *reinterpret_cast<uint4*>(rowp + ((c ^ (r & 7)) << 4)) =
            make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
      }
    } else {
      // 32 columns = 128 bytes: all 8 chunks of box cc
      uint8_t* rowp = st + cc * 16384 + r * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<float4*>(rowp + ((c ^ (r & 7)) << 4)) =
            make_float4(__uint_as_float(v[4 * c]) * mul, __uint_as_float(v[4 * c + 1]) * mul,
                        __uint_as_float(v[4 * c + 2]) * mul, __uint_as_float(v[4 * c + 3]) * mul);
    }
  }
}

struct BwdParams {
  CUtensorMap tq, tdo;         // [B*Hq][N][d] bf16, box {64, MQ}, 128B swizzle
  CUtensorMap tk, tv;          // [B*Hkv][N][d] bf16, box {64, 128}
  CUtensorMap tdq;             // [B*Hq][N][d] fp32, box {32, MQ}, 128B swizzle (reduce-add)
  CUtensorMap tdk, tdv;        // [B*Hkv][N][d] grad dtype, box {128 bytes, 128}, 128B swizzle
  const float* lse2;           // [B*Hq][Npad]
  const float* dvec;           // [B*Hq][Npad]
  void* dK;
  void* dV;
  const uint8_t* mask;
  unsigned* err;
  int N, Npad, Hq, Hkv, nb, causal, grad_bf16, BHk;
  MaskMod mod;                 // keys each query sees (the causal flag is its wr = 0)
  float c;                     // scale * log2(e)
  float cap1, cap2;            // soft-capping: scores in log2 units = cap1 * tanh(cap2 * q.k)
  float scale;
  const int* cu;               // variable-length batch: sequence offsets [B+1], or null
  int total;                   // packed rows (variable-length batch)
  int no_dq;                   // skip dQ (the deterministic dQ kernel computes it)
  long long stall;             // > 0: injected wait of this many cycles (test hook)
};

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) break;
  }
}

template <int D, bool kVarlen, bool kCap>
__global__ void __launch_bounds__(Cfg<D>::kThreads, 1) bwd_kernel(const __grid_constant__ BwdParams p) {
  using C = Cfg<D>;
  constexpr int MQ = C::MQ;
  extern __shared__ uint8_t smem_raw[];
  Ctl& ctl = *reinterpret_cast<Ctl*>(smem_raw);
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base_addr = (raw_addr + sizeof(Ctl) + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_addr - raw_addr);
  float* vec = reinterpret_cast<float*>(base + C::kOffVec);

  // KV heads are taken kChunk at a time (their Q/dO stay in L2 during a
  // wave); inside a chunk the low key tiles, which see the most query tiles
  // under the causal flag, start first.
  int bhk, kb;
  chunked_order(blockIdx.x, p.nb, p.BHk, kChunk, bhk, kb);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = kb * kBN;
  const int b = bhk / p.Hkv, hk = bhk % p.Hkv;
  const int grp = p.Hq / p.Hkv;
  // Dense: rows 0..N-1 of plane (b, head). Variable-length batch: sequence b
  // is rows cu[b] .. cu[b+1]-1 of the packed tensors (planes are heads); key
  // tiles past its end have nothing to do. Offsets are clamped to [0, total].
  int N = p.N, row0 = 0;
  if constexpr (kVarlen) {
    const int s0 = min(max(p.cu[b], 0), p.total);
    const int s1 = min(max(p.cu[b + 1], s0), p.total);
    N = min(s1 - s0, p.N);
    if (n0 >= N) return;
    row0 = s0;
  }
  const int kplane = kVarlen ? hk : bhk;

  if (threadIdx.x == 0) {
    // A launch whose error word is already set (an earlier wait ran out and
    // nobody has read the word yet) does no work: its inputs may be invalid.
    // This one thread reads the word (while it sets up the barriers) and the
    // whole CTA leaves together after the block barrier below, before any
    // wait.
    const unsigned err_word = *reinterpret_cast<volatile unsigned*>(p.err);
    mbar_init(&ctl.kv_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&ctl.qdo_full[s], 1);
      mbar_init(&ctl.qdo_empty[s], 1);
    }
    mbar_init(&ctl.sp_full[0], 1);
    mbar_init(&ctl.sp_full[1], 1);
    mbar_init(&ctl.p_ready[0], C::kItemSplit ? 4 : C::kSoftWarps);
    mbar_init(&ctl.p_ready[1], C::kItemSplit ? 4 : C::kSoftWarps);
    mbar_init(&ctl.dq_full, 1);
    mbar_init(&ctl.dq_free, 4);
    mbar_init(&ctl.acc_done, 1);
    mbar_init(&ctl.never, 1);
    ctl.abort = 0;
    fence_mbar_init();
    {
      // This thread is also the TMA producer: the K and V tiles start now, so
      // their latency (and that of the error-word read) overlaps the TMEM
      // allocation, the query-tile list and the block barrier. A CTA that
      // then finds the word set waits for them to land and does nothing else.
      prefetch_tmap(&p.tk);
      prefetch_tmap(&p.tv);
      mbar_expect_tx(&ctl.kv_full, 2 * C::kKVBytes);
      for (int cb = 0; cb < D / 64; ++cb) {
        tma_load_3d(base + C::kOffK + cb * kBN * 128, &p.tk, &ctl.kv_full, cb * 64, row0 + n0,
                    kplane);
        tma_load_3d(base + C::kOffV + cb * kBN * 128, &p.tv, &ctl.kv_full, cb * 64, row0 + n0,
                    kplane);
      }
    }
    ctl.skip = err_word != 0u;
  }
  if (warp == 2) {
    tmem_alloc(&ctl.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 3) {
    // Query tiles that can see this key tile, in increasing order (entries
    // flagged kFullBit see all of it).
    const int nqt = (N + MQ - 1) / MQ;
    // first query tile whose rows can reach this key tile
    const int qt_lo = mod_first_query(p.mod, n0) / MQ;
    int count = 0;
    for (int t0 = qt_lo; t0 < nqt; t0 += 32) {
      const int qt = t0 + lane;
      int cls = kTileEmpty;
      if (qt < nqt && (!p.mask || p.mask[(size_t)((qt * MQ) / 128) * p.nb + kb]))
        cls = mod_classify(p.mod, qt * MQ, qt * MQ + MQ - 1, n0, n0 + kBN - 1, N);
      const bool vis = cls != kTileEmpty;
      const unsigned bal = __ballot_sync(0xffffffffu, vis);
      if (vis)
        ctl.qtiles[count + __popc(bal & ((1u << lane) - 1u))] =
            static_cast<uint16_t>(qt | (cls == kTileFull ? kFullBit : 0));
      count += __popc(bal);
    }
    if (lane == 0) ctl.nq = count;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = ctl.tmem_base;
  if (ctl.skip) {   // the error word was set at launch: no work
    if (threadIdx.x == 0) drain_wait(&ctl.kv_full, 0);
    if (warp == 2) tmem_dealloc(tm, 512);
    return;
  }
  const int nq = ctl.nq;
  const int n_items = nq * grp;
  const Guard g{&ctl.abort, p.err};
  constexpr int kChunks = MQ / 32 / C::kColHalves;   // 32-column chunks per softmax warp
  static_assert(kChunks == 2, "the MMA warp waits on two chunk steps per item");
  // item i -> (query head, first query row)
  auto item_bh = [&](int i) { return b * p.Hq + hk * grp + i / nq; };
  // TMA plane of item i's Q / dO / dQ rows
  auto item_plane = [&](int i) { return kVarlen ? hk * grp + i / nq : item_bh(i); };
  auto item_q0 = [&](int i) { return static_cast<int>(ctl.qtiles[i % nq] & ~kFullBit) * MQ; };
  // TMEM columns of item i
  auto s_col = [&](int i) { return (i & 1) ? C::kS1 : C::kS0; };
  auto dp_col = [&](int i) { return (i & 1) ? C::kDP1 : C::kDP0; };
  auto dq_col = [&](int i) { return C::kDbl ? s_col(i) : C::kDQ; };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // (K and V were issued before the block barrier.)
      prefetch_tmap(&p.tq);
      prefetch_tmap(&p.tdo);
      int issued = 0;
      for (int i = 0; i < n_items; ++i) {
        const int s = i % C::kStages;
        if (i >= C::kStages && !mbar_wait(&ctl.qdo_empty[s], ((i / C::kStages) - 1) & 1, g)) break;
        const int bh = item_bh(i), q0 = item_q0(i), pl = item_plane(i);
        mbar_expect_tx(&ctl.qdo_full[s], 2 * C::kQBytes + 2 * MQ * 4);
        for (int cb = 0; cb < D / 64; ++cb) {
          tma_load_3d(base + C::kOffQ + s * C::kQBytes + cb * C::kQBlock, &p.tq,
                      &ctl.qdo_full[s], cb * 64, row0 + q0, pl);
          tma_load_3d(base + C::kOffDO + s * C::kQBytes + cb * C::kQBlock, &p.tdo,
                      &ctl.qdo_full[s], cb * 64, row0 + q0, pl);
        }
        const size_t vo = (size_t)bh * p.Npad + q0;
        bulk_load(vec + (s * 2 + 0) * MQ, p.lse2 + vo, MQ * 4, &ctl.qdo_full[s]);
        bulk_load(vec + (s * 2 + 1) * MQ, p.dvec + vo, MQ * 4, &ctl.qdo_full[s]);
        issued = i + 1;
      }
      drain_wait(&ctl.kv_full, 0);
      for (int s = 0; s < C::kStages && s < issued; ++s)
        drain_wait(&ctl.qdo_full[s], (((issued - 1 - s) / C::kStages + 1) - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_items > 0) {
      constexpr uint32_t idSP = idesc_bf16(kBN, MQ, false, false);   // K-major A and B
      constexpr uint32_t idKV = idesc_bf16(kBN, D, false, true);     // B MN-major
      constexpr uint32_t idQ = idesc_bf16(128, 64, true, true);      // both MN-major
      // Base descriptors, built once (K-major and MN-major readings of K, V,
      // the Q / dO ring and the dS^T buffers); each operand below is one of
      // them plus a byte offset (sdesc_at).
      const uint32_t ka = smem_u32(base + C::kOffK), va = smem_u32(base + C::kOffV);
      const uint32_t qa = smem_u32(base + C::kOffQ), da = smem_u32(base + C::kOffDO);
      const uint32_t dsa = smem_u32(base + C::kOffDS);
      const uint64_t dK_k = sdesc_sw128(ka, 16, 1024), dV_k = sdesc_sw128(va, 16, 1024);
      const uint64_t dQ_k = sdesc_sw128(qa, 16, 1024), dO_k = sdesc_sw128(da, 16, 1024);
      const uint64_t dQ_mn = sdesc_sw128(qa, C::kQBlock, 1024);
      const uint64_t dO_mn = sdesc_sw128(da, C::kQBlock, 1024);
      const uint64_t dS_k = sdesc_sw128(dsa, 16, 1024);
      const uint64_t dK_mn = sdesc_sw128(ka, kBN * 128, 1024);
      const uint64_t dS_mn = sdesc_sw128(dsa, kBN * 128, 1024);
      auto qoff = [&](int i) { return (uint32_t)((i % C::kStages) * C::kQBytes); };
      auto dsoff = [&](int i) { return (uint32_t)((i & 1) * C::kDSBytes); };
      auto issue_s = [&](int i) {   // S^T = K Q_i^T
        const uint64_t dq = sdesc_at(dQ_k, qoff(i));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tm + s_col(i), sdesc_at(dK_k, (kk >> 2) * (kBN * 128) + (kk & 3) * 32),
                 sdesc_at(dq, (kk >> 2) * C::kQBlock + (kk & 3) * 32), idSP, kk > 0);
      };
      auto issue_dp = [&](int i) {  // dP^T = V dO_i^T
        const uint64_t ddo = sdesc_at(dO_k, qoff(i));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tm + dp_col(i), sdesc_at(dV_k, (kk >> 2) * (kBN * 128) + (kk & 3) * 32),
                 sdesc_at(ddo, (kk >> 2) * C::kQBlock + (kk & 3) * 32), idSP, kk > 0);
      };
      // dV += P^T dO_i and dK += dS^T Q_i over the query columns the softmax
      // warps finished in chunk step `st` (32-column chunk cc = h * kChunks + st
      // of each column half h; 16-query k-steps 2cc and 2cc + 1).
      auto issue_dv = [&](int i, int st) {  // P^T bf16 in the S columns
        const uint64_t ddo = sdesc_at(dO_mn, qoff(i));
#pragma unroll
        for (int h = 0; h < C::kColHalves; ++h)
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {
            const int kk = 2 * (h * kChunks + st) + k2;
            mma_ts(tm + C::kDV, tm + s_col(i) + (kk >> 1) * 32 + (kk & 1) * 8,
                   sdesc_at(ddo, kk * 2048), idKV, (i > 0 || kk > 0));
          }
      };
      auto issue_dk = [&](int i, int st) {
        const uint64_t dq = sdesc_at(dQ_mn, qoff(i)), ds = sdesc_at(dS_k, dsoff(i));
#pragma unroll
        for (int h = 0; h < C::kColHalves; ++h)
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {
            const int kk = 2 * (h * kChunks + st) + k2;
            mma_ss(tm + C::kDK, sdesc_at(ds, (kk >> 2) * (kBN * 128) + (kk & 3) * 32),
                   sdesc_at(dq, kk * 2048), idKV, (i > 0 || kk > 0));
          }
      };
      auto issue_dq = [&](int i) {  // dQ_i^T = K^T dS_i^T (d = 128) or dQ_i = dS_i K (d = 64)
        const uint64_t ds = sdesc_at(dS_mn, dsoff(i));
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          if constexpr (D == 128)
            mma_ss(tm + dq_col(i), sdesc_at(dK_mn, kk * 2048), sdesc_at(ds, kk * 2048), idQ, kk > 0);
          else
            mma_ss(tm + dq_col(i), sdesc_at(ds, kk * 2048), sdesc_at(dK_mn, kk * 2048), idQ, kk > 0);
        }
      };
      // (normally landed long before: the phase is tested before the abort
      // flag is read)
      auto wait_q = [&](int i) {
        return mbar_wait_ready_first(&ctl.qdo_full[i % C::kStages], (i / C::kStages) & 1, g);
      };
      bool ok = injected_stall(&ctl.never, p.stall, g) && mbar_wait(&ctl.kv_full, 0, g) &&
                wait_q(0);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
        mma_commit(&ctl.sp_full[0]);
      }
      if constexpr (C::kDbl) {
        if (ok && n_items > 1 && (ok = wait_q(1))) {
          tc_fence_after();
          issue_s(1);
          issue_dp(1);
          mma_commit(&ctl.sp_full[1]);
        }
        for (int i = 0; ok && i < n_items; ++i) {
          // d = 128: one signal per item (per-chunk signals measured slower),
          // on p_ready[i & 1]. Two barriers by item parity: S(i+1) is ready
          // while item i's softmax runs, so a fast warp may arrive for item
          // i+1 before a slow one arrives for item i; on one barrier that
          // arrival could complete item i's phase early. Item i+2 cannot
          // start before item i's phase completes (S(i+2) waits for dQ(i)).
          if (!(ok = mbar_wait(&ctl.p_ready[i & 1], (i >> 1) & 1, g))) break;
          tc_fence_after();
          issue_dv(i, 0);
          issue_dv(i, 1);
          issue_dk(i, 0);
          issue_dk(i, 1);
          mma_commit(&ctl.qdo_empty[i % C::kStages]);
          if (!p.no_dq) {
            issue_dq(i);
            mma_commit(&ctl.dq_full);
          }
          if (i + 2 < n_items) {
            // (checked here, not before P(i): item i+2's tiles are often
            // still landing when P(i) is ready; measured 4 % slower there)
            if (!(ok = wait_q(i + 2))) break;
            tc_fence_after();
            issue_dp(i + 2);
            if (!p.no_dq && !(ok = mbar_wait(&ctl.dq_free, i & 1, g))) break;   // dQ(i) drained
            tc_fence_after();
            issue_s(i + 2);
            mma_commit(&ctl.sp_full[i & 1]);
          }
        }
      } else {
        for (int i = 0; ok && i < n_items; ++i) {
          // Q / dO of item i+1 (loaded once item i-1 freed its stage) are
          // checked before P(i), so that nothing but the P signals sits
          // between item i's MMAs and those of item i+1.
          if (!(ok = (i + 1 >= n_items || wait_q(i + 1)) && mbar_wait(&ctl.p_ready[0], i & 1, g)))
            break;
          tc_fence_after();
          issue_dv(i, 0);
          issue_dk(i, 0);
          if (!(ok = mbar_wait(&ctl.p_ready[1], i & 1, g))) break;
          tc_fence_after();
          issue_dv(i, 1);
          if (i + 1 < n_items) {
            issue_s(i + 1);
            issue_dp(i + 1);
            mma_commit(&ctl.sp_full[0]);
          }
          issue_dk(i, 1);
          mma_commit(&ctl.qdo_empty[i % C::kStages]);
          if (!p.no_dq) {
            if (i > 0 && !(ok = mbar_wait(&ctl.dq_free, (i - 1) & 1, g))) break;
            tc_fence_after();
            issue_dq(i);
            mma_commit(&ctl.dq_full);
          }
        }
      }
      mma_commit(&ctl.acc_done);
      drain_wait(&ctl.acc_done, 0);
    }
  } else if (warp >= 4 && warp < 4 + C::kSoftWarps) {
    // ------------------------------------------------------------ softmax / dS
    // d = 64: warps 4-7 take the first half of each item's query columns and
    // warps 8-11 the second half. d = 128: warps 4-7 take the even items and
    // warps 8-11 the odd ones (with FA_BWD_ITEM_SPLIT=0, warps 4-7 take all).
    const int wq = warp & 3;
    const int half = (warp - 4) >> 2;
    const int i_first = C::kItemSplit ? half : 0, i_step = C::kItemSplit ? 2 : 1;
    const int col_half = C::kItemSplit ? 0 : half;
    const int r = wq * 32 + lane;                 // key row inside the tile
    const int kv = n0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float c = p.c;
    // queries that see this thread's key: [qlo, qhi] (empty past N)
    int qlo, qhi;
    mod_key_queries(p.mod, kv, N, qlo, qhi);
    for (int i = i_first; i < n_items; i += i_step) {
      const int s = i % C::kStages;
      const bool spok = C::kDbl ? mbar_wait(&ctl.sp_full[i & 1], (i >> 1) & 1, g)
                                : mbar_wait(&ctl.sp_full[0], i & 1, g);
      if (!spok) break;
      if (!mbar_wait_ready_first(&ctl.qdo_full[s], (i / C::kStages) & 1, g)) break;
      tc_fence_after();
      const int q0 = item_q0(i);
      const bool need_mask = !(ctl.qtiles[i % nq] & kFullBit);
      const float* lse_s = vec + (s * 2 + 0) * MQ;
      const float* d_s = vec + (s * 2 + 1) * MQ;
      uint8_t* dsrow = base + C::kOffDS + (i & 1) * C::kDSBytes + r * 128;
#pragma unroll 1
      for (int ch = 0; ch < kChunks; ++ch) {
        const int cc = col_half * kChunks + ch;
        uint32_t sv[32], dp[32];
        tmem_ld32x2(tm + s_col(i) + lane_off + cc * 32, tm + dp_col(i) + lane_off + cc * 32, sv,
                    dp);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int qa_ = q0 + cc * 32 + e;
          const float4 l2 = *reinterpret_cast<const float4*>(lse_s + ((cc * 32 + e) & ~3));
          const float4 dd = *reinterpret_cast<const float4*>(d_s + ((cc * 32 + e) & ~3));
          const float la = (e & 2) ? l2.z : l2.x, lb = (e & 2) ? l2.w : l2.y;
          const float da_ = (e & 2) ? dd.z : dd.x, db_ = (e & 2) ? dd.w : dd.y;
          // soft-capping: P from the capped score, and dS picks up the
          // derivative of the cap, 1 - tanh^2
          float t0 = 0.f, t1 = 0.f;
          if constexpr (kCap) {
            t0 = tanh_ex2(__uint_as_float(sv[e]) * p.cap2);
            t1 = tanh_ex2(__uint_as_float(sv[e + 1]) * p.cap2);
          }
          float p0 = kCap ? ex2(fmaf(t0, p.cap1, -la)) : ex2(fmaf(__uint_as_float(sv[e]), c, -la));
          float p1 =
              kCap ? ex2(fmaf(t1, p.cap1, -lb)) : ex2(fmaf(__uint_as_float(sv[e + 1]), c, -lb));
          if (need_mask) {
            if (qa_ < qlo || qa_ > qhi) p0 = 0.f;
            if (qa_ + 1 < qlo || qa_ + 1 > qhi) p1 = 0.f;
          }
          float g0 = p0 * (__uint_as_float(dp[e]) - da_);
          float g1 = p1 * (__uint_as_float(dp[e + 1]) - db_);
          if constexpr (kCap) {
            g0 *= fmaf(-t0, t0, 1.f);
            g1 *= fmaf(-t1, t1, 1.f);
          }
          pk[e >> 1] = pack_bf16(p0, p1);
          dk[e >> 1] = pack_bf16(g0, g1);
        }
        // P^T (bf16 pairs) into the first 16 of this chunk's own 32 S columns,
        // which this thread has already read; no other warp reads them
        tmem_st16(tm + s_col(i) + lane_off + cc * 32, pk);
        // dS^T row into the 128B-swizzled K-major buffer: 16-byte chunks of 8 values
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int qc = cc * 32 + k * 8;               // first query column of the chunk
          const int blk = qc >> 6, c16 = (qc & 63) >> 3;
          uint4 v = make_uint4(dk[k * 4 + 0], dk[k * 4 + 1], dk[k * 4 + 2], dk[k * 4 + 3]);
          *reinterpret_cast<uint4*>(dsrow + blk * (kBN * 128) + ((c16 ^ (r & 7)) << 4)) = v;
        }
        // This chunk's P^T and dS^T are complete: for d = 64 the MMA warp
        // may run the dV and dK steps over its query columns now (p_ready[ch];
        // item i+1's S is issued only after both steps of item i, so no warp
        // runs an item ahead); for d = 128 it waits for the whole item (one
        // signal after the last chunk, on p_ready[i & 1]).
        if (C::kColHalves == 2 || ch == kChunks - 1) {
          tmem_st_wait();
          fence_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl.p_ready[C::kDbl ? (i & 1) : ch]);
        }
      }
    }
    // ------------------------------------------------------------ dK, dV epilogue
    if (n_items > 0) {
      mbar_wait(&ctl.acc_done, 0, g);
      tc_fence_after();
    }
    const bool valid = kv < N;
    // 8 softmax warps: warps 4-7 store dK, warps 8-11 dV. 4 (d = 128): warps
    // 4-7 store dK and the dQ drain warps dV (both for packed batches).
    const int which_lo = (C::kSoftWarps == 8) ? half : 0;
    const int which_hi = (C::kSoftWarps == 8) ? half + 1 : (!kVarlen && C::kDrainDV ? 1 : 2);
    if constexpr (!kVarlen) {
      // dK (and dV) through the shared memory of the Q/dO ring and the dS
      // buffers (every MMA has completed): dK at the start, dV one staged
      // tensor after it. Each warpgroup's first thread then stores its
      // tensor's whole lines with TMA (rows at or past N are clipped by the
      // tensor map).
      const int esz = p.grad_bf16 ? 2 : 4;
      const int tbytes = kBN * D * esz;   // one staged tensor
#pragma unroll 1
      for (int which = which_lo; which < which_hi; ++which)
        stage_grad<D>(base + C::kOffQ + which * tbytes, tm + (which ? C::kDV : C::kDK) + lane_off,
                      n_items > 0, which ? 1.f : p.scale, p.grad_bf16, r);
      fence_async_smem();
      named_sync(2 + half, 128);
      if (wq == 0 && lane == 0) {
        const int boxes = D * esz / 128, box_cols = 128 / esz;
        for (int which = which_lo; which < which_hi; ++which)
          for (int bx = 0; bx < boxes; ++bx)
            tma_store_3d(which ? &p.tdv : &p.tdk, base + C::kOffQ + which * tbytes + bx * 16384,
                         bx * box_cols, n0, bhk);
        bulk_commit();
        bulk_wait_read0();   // the staging is read before the CTA exits
      }
    } else {
      // packed batch: a 128-row box could reach into the next sequence, so
      // rows are stored one by one ([total][Hkv][d])
      const size_t orow = ((size_t)(row0 + (valid ? kv : 0)) * p.Hkv + hk) * D;
#pragma unroll 1
      for (int which = which_lo; which < which_hi; ++which) {
        const uint32_t col = which ? C::kDV : C::kDK;
        const float mul = which ? 1.f : p.scale;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t v[32];
          if (n_items > 0) {
            tmem_ld32(tm + col + lane_off + cc * 32, v);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0u;
          }
          if (!valid) continue;
          if (p.grad_bf16) {
            __nv_bfloat16* out = static_cast<__nv_bfloat16*>(which ? p.dV : p.dK) + orow + cc * 32;
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              w[e] = pack_bf16(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              reinterpret_cast<uint4*>(out)[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2],
                                                            w[4 * e + 3]);
          } else {
            float* out = static_cast<float*>(which ? p.dV : p.dK) + orow + cc * 32;
#pragma unroll
            for (int e = 0; e < 8; ++e)
              reinterpret_cast<float4*>(out)[e] =
                  make_float4(__uint_as_float(v[4 * e]) * mul, __uint_as_float(v[4 * e + 1]) * mul,
                              __uint_as_float(v[4 * e + 2]) * mul,
                              __uint_as_float(v[4 * e + 3]) * mul);
          }
        }
      }
    }
  } else if (warp >= 4 + C::kSoftWarps) {
    // ------------------------------------------------------------ dQ drain
    const int wq = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const bool leader = (warp == 4 + C::kSoftWarps && lane == 0);
    uint8_t* stg = base + C::kOffStg;
    const float sc = p.scale;
    // Every drain thread runs all iterations (waits return at once after an
    // abort), so the named barriers below always see all 128 threads.
    const int n_drain = p.no_dq ? 0 : n_items;
    for (int i = 0; i < n_drain; ++i) {
      mbar_wait(&ctl.dq_full, i & 1, g);
      tc_fence_after();
      uint32_t v[64];
      tmem_ld64(tm + dq_col(i) + lane_off, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.dq_free);
      const int pl = item_plane(i), q0 = row0 + item_q0(i);
      if constexpr (D == 128) {
        // lane = head-dim column d = 32*wq + lane; v[q] for q = 0..63. Two
        // 16 KB halves: warps 0-1 stage d 0..63, then warps 2-3 stage 64..127.
        uint8_t* box = stg + (wq & 1) * C::kStgBox + (lane & 3) * 4;
        const int ch = lane >> 2;
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {
          if (leader) bulk_wait_read0();   // the previous reduce has read the staging
          named_sync(1, 128);
          if ((wq >> 1) == hf) {
#pragma unroll
            for (int q = 0; q < MQ; ++q)
              *reinterpret_cast<float*>(box + q * 128 + ((ch ^ (q & 7)) << 4)) =
                  __uint_as_float(v[q]) * sc;
            fence_async_smem();
          }
          named_sync(1, 128);
          if (leader) {
            tma_reduce_add_3d(&p.tdq, stg, (2 * hf) * 32, q0, pl);
            tma_reduce_add_3d(&p.tdq, stg + C::kStgBox, (2 * hf + 1) * 32, q0, pl);
            bulk_commit();
          }
        }
      } else {
        // lane = query row q = 32*wq + lane; v[d] for d = 0..63
        if (leader) bulk_wait_read0();
        named_sync(1, 128);
        const int q = wq * 32 + lane;
#pragma unroll
        for (int bx = 0; bx < 2; ++bx)
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int d0 = bx * 32 + k * 4;
            *reinterpret_cast<float4*>(stg + bx * C::kStgBox + q * 128 + ((k ^ (q & 7)) << 4)) =
                make_float4(__uint_as_float(v[d0]) * sc, __uint_as_float(v[d0 + 1]) * sc,
                            __uint_as_float(v[d0 + 2]) * sc, __uint_as_float(v[d0 + 3]) * sc);
          }
        fence_async_smem();
        named_sync(1, 128);
        if (leader) {
#pragma unroll
          for (int bx = 0; bx < D / 32; ++bx)
            tma_reduce_add_3d(&p.tdq, stg + bx * C::kStgBox, bx * 32, q0, pl);
          bulk_commit();
        }
      }
    }
    if constexpr (!kVarlen && C::kDrainDV) {
      // dV epilogue, beside the softmax warps' dK: staged one tensor after
      // dK, clear of the dQ staging
      if (n_items > 0) {
        mbar_wait(&ctl.acc_done, 0, g);
        tc_fence_after();
      }
      const int esz = p.grad_bf16 ? 2 : 4;
      const int tbytes = kBN * D * esz;
      stage_grad<D>(base + C::kOffQ + tbytes, tm + C::kDV + lane_off, n_items > 0, 1.f,
                    p.grad_bf16, wq * 32 + lane);
      fence_async_smem();
      named_sync(1, 128);
      if (leader) {
        const int boxes = D * esz / 128, box_cols = 128 / esz;
        for (int bx = 0; bx < boxes; ++bx)
          tma_store_3d(&p.tdv, base + C::kOffQ + tbytes + bx * 16384, bx * box_cols, n0, bhk);
        bulk_commit();
      }
    }
    if (leader) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

template <int D>
cudaError_t launch(const Problem& pr) {
  using C = Cfg<D>;
  BwdParams kp;
  memset(&kp, 0, sizeof(kp));
  const uint64_t BHq = (uint64_t)pr.B * pr.Hq, BHk = (uint64_t)pr.B * pr.Hkv;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_seq_tmap(&kp.tq, pr, pr.Q, bf, 2, pr.Hq, 64, C::MQ, sw) ||
      !make_seq_tmap(&kp.tdo, pr, pr.dO, bf, 2, pr.Hq, 64, C::MQ, sw) ||
      !make_seq_tmap(&kp.tk, pr, pr.K, bf, 2, pr.Hkv, 64, kBN, sw) ||
      !make_seq_tmap(&kp.tv, pr, pr.V, bf, 2, pr.Hkv, 64, kBN, sw) ||
      !make_seq_tmap(&kp.tdq, pr, pr.dQacc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, pr.Hq, 32, C::MQ,
                     sw))
    return cudaErrorInvalidValue;
  {
    // dK / dV epilogue (dense batches): boxes of 128 bytes x 128 rows
    const bool gb = pr.grad_dtype == 1;
    const auto gt = gb ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const int es = gb ? 2 : 4;
    if (!pr.cu && (!make_seq_tmap(&kp.tdk, pr, pr.dK, gt, es, pr.Hkv, 128 / es, kBN, sw) ||
                   !make_seq_tmap(&kp.tdv, pr, pr.dV, gt, es, pr.Hkv, 128 / es, kBN, sw)))
      return cudaErrorInvalidValue;
  }
  kp.lse2 = pr.LSE2ws;
  kp.dvec = pr.Dws;
  kp.dK = pr.dK;
  kp.dV = pr.dV;
  kp.mask = pr.mask;
  kp.err = pr.err;
  kp.N = pr.N;
  kp.Npad = pr.Npad;
  kp.Hq = pr.Hq;
  kp.Hkv = pr.Hkv;
  kp.nb = pr.nb;
  kp.causal = pr.causal;
  kp.mod = mask_mod_of(pr);
  kp.cap1 = pr.softcap > 0.f ? pr.softcap * kLog2e : 0.f;
  kp.cap2 = pr.softcap > 0.f ? pr.scale / pr.softcap : 0.f;
  kp.grad_bf16 = pr.grad_dtype == 1;
  kp.c = pr.scale * kLog2e;
  kp.scale = pr.scale;
  kp.cu = pr.cu;
  kp.total = pr.total;
  kp.no_dq = pr.no_dq;
  kp.stall = debug_stall_cycles(kStallBwd);
  const size_t smem = sizeof(Ctl) + 1024 + C::kOffEnd;
  for (const void* f : {(const void*)bwd_kernel<D, false, false>,
                        (const void*)bwd_kernel<D, true, false>,
                        (const void*)bwd_kernel<D, false, true>}) {
    const cudaError_t e = set_max_dynamic_smem(f, (int)smem);
    if (e != cudaSuccess) return e;
  }
  kp.BHk = (int)BHk;
  dim3 grid((unsigned)(BHk * pr.nb));
  const bool cap = pr.softcap > 0.f;
  if (pr.cu && cap) return cudaErrorInvalidValue;   // not offered for packed batches
  if (pr.cu)
    bwd_kernel<D, true, false><<<grid, C::kThreads, smem, pr.stream>>>(kp);
  else if (cap)
    bwd_kernel<D, false, true><<<grid, C::kThreads, smem, pr.stream>>>(kp);
  else
    bwd_kernel<D, false, false><<<grid, C::kThreads, smem, pr.stream>>>(kp);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

bool sm100_bwd_supported(const Problem& p) {
  const int mq = (p.d == 64) ? 128 : 64;
  return p.dtype == 1 && (p.d == 64 || p.d == 128) && p.scale > 0.f &&
         (p.N + mq - 1) / mq <= kMaxQTiles && (long long)p.B * p.Hkv * p.nb < (1ll << 31) &&
         (long long)p.B * p.Hkv < (1ll << 31);
}

// dQ is accumulated in fp32 by TMA reduce-adds: into dQ itself for fp32
// gradients, into the workspace accumulator (then converted) for bf16.
bool sm100_bwd_uses_dq_accumulator(const Problem& p) { return p.grad_dtype == 1; }

cudaError_t sm100_bwd_main(const Problem& p) {
  return p.d == 64 ? launch<64>(p) : launch<128>(p);
}

}  // namespace fa
