// Fused attention forward for sm_100a: tcgen05 MMAs with TMEM accumulators,
// TMA-fed K/V ring, warp-specialised producer / MMA / softmax warps.
//
// Computes, for each query row, O = softmax(scale * Q K^T) V over the visible
// keys and LSE = logsumexp(scale * Q K^T) (FlashAttention lesson, Researcher
// section "The problem being solved"), never writing S or P to HBM (paper
// summary, "Core Idea" items 1, 2 and 4). Each CTA owns two 128-row query tiles
// of one (batch, head) and walks the key tiles either needs (K and V are loaded
// once for both); for each key tile j:
//
//   S_t = Q_t K_j^T             tcgen05.mma, A and B from shared memory, S in TMEM
//   online softmax on S_t       one thread per row (tcgen05.ld 32x32b), base-2
//                               exponentials with scale*log2(e) folded in
//   O_t += P_t V_j              tcgen05.mma, P (bf16) from TMEM, V from shared memory
//
// The running statistics follow the Researcher section's "Online softmax"
// recurrence: m^(j) = max(m^(j-1), rowmax S^(j)), l^(j) = e^(m^(j-1)-m^(j))
// l^(j-1) + rowsum e^(S^(j)-m^(j)), and O^(j) likewise. The kernel keeps a
// reference maximum per row and moves it (rescaling l and the TMEM
// accumulator together, the "correction" step) only when a tile's row maximum
// exceeds it by more than 2^8 in the exponent; between moves the terms are
// taken relative to the unchanged reference. The recurrence holds for any
// reference value, so O^(T)/l^(T) is unchanged; the bound keeps every P term
// <= 256 (no overflow in fp32 or bf16) and skips most TMEM round trips.
//
// Two query tiles alternate on the tensor core (ping-pong): while one
// softmax warpgroup works on S_0, the MMA warp runs P_1 V and Q_1 K^T, and the
// other way round. Each softmax signals twice per tile: once P of the first
// 64 keys is in TMEM (the MMA warp starts P V on those keys) and once all of
// P is; a rescale of O, when the reference max moved, happens before the
// first signal. P_t is written into the upper half of S_t's TMEM columns;
// tcgen05.mma operations issued by one thread execute in order, so the next
// Q_t K^T that overwrites S_t cannot overtake the P_t V that reads it.
//
// A key tile one query tile sees nothing of (a block-mask cell that is off,
// a window edge, the causal diagonal of the other tile) is either computed for
// it fully masked, keeping the two tiles in lockstep (dense, causal and
// variable-length launches, where there are at most one or two such tiles per
// CTA), or skipped for it: no Q K^T, softmax or P V (kSkip: windows with a
// left edge and documents). The skipping form counts barrier phases per query
// tile; measured on B200 it is 4-12% slower than the lockstep form where
// nearly every tile is seen by both query tiles, hence the two forms.
//
// Forms per launch: the persistent form of the lockstep kernel (one CTA per
// SM drawing two-tile items from a queue) for dense and causal launches up to
// FA_FWD_PERSIST_MAXN keys; the one-item lockstep form above that and for
// variable-length batches; the skipping form for left window edges and
// documents; and, for block masks, the split form (one query tile per CTA,
// its visible key tiles dealt to the two softmax warpgroups, the two partial
// results merged by their log-sum-exp).
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 MMA issuer, warp 2
// TMEM allocator, warp 3 builds the key-tile list, warps 4-7 softmax of query
// tile 0, warps 8-11 softmax of query tile 1.
#include <math.h>

#include <algorithm>
#include <utility>

#include "sm100_common.cuh"

namespace fa {
namespace {
using namespace sm100;

constexpr int kBM = 128;           // query rows per tile
constexpr int kBN = 128;           // keys per tile
constexpr int kMaxTiles = 2048;    // key tiles per sequence: N <= 262144
constexpr int kThreads = 384;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kTau = 8.0f;       // reference-max slack, log2 units
constexpr int kMaxChunk = 16;      // most heads interleaved in launch order

constexpr int kMaxSlots = 10;     // most K/V ring slots of any form

// Build-time tuning (defaults measured on B200): K/V ring slots of the
// lockstep form at d = 128, and the FMA-pipe share of the softmax
// exponentials in eighths at d = 64 and d = 128.
#ifndef FA_FWD_SLOTS_D128
#define FA_FWD_SLOTS_D128 5
#endif
#ifndef FA_FWD_EMU_PAIRS_D64
#define FA_FWD_EMU_PAIRS_D64 0
#endif
#ifndef FA_FWD_EMU_PAIRS_D128
#define FA_FWD_EMU_PAIRS_D128 0
#endif
// Dense and causal launches with N up to this many keys run the persistent
// form (one CTA per SM over a queue of items), the others one CTA per item:
// measured on B200, the persistent form is 1-13% faster up to N = 4096 (the
// fixed cost per item matters most there) and 3-6% slower at 8K-16K (its
// steady state is a little slower). 0: never persistent.
// Block-sparse launches (a block mask given) run the split form: bit 0 at
// d = 64, bit 1 at d = 128; otherwise the paired skipping form. Bit 2: every
// launch of the skipping form (windows, documents) runs the split form too.
#ifndef FA_FWD_SPLIT
#define FA_FWD_SPLIT 3
#endif
#ifndef FA_FWD_PERSIST_MAXN
#define FA_FWD_PERSIST_MAXN 4096
#endif

template <int D, bool kSkip>
struct Cfg {
  // K and V tiles share one ring of slots, loaded in the order they are
  // consumed (K_0, V_0, K_1, V_1, ...) and released one by one (K_j once the
  // last S MMA that reads it has completed, V_j after the last P V), so the
  // load of K_{j+3} can start while iteration j is still running. The
  // lockstep form keeps no tile lists and spends that shared memory on more
  // slots: 5 x 32 KB at d = 128 (plus 64 KB of Q: 224 KB).
  static constexpr int kSlots =
      kSkip ? ((D == 64) ? 8 : 4) : ((D == 64) ? 10 : FA_FWD_SLOTS_D128);
  // Share of the softmax exponentials computed on the FMA pipe, in eighths
  // (tiles without masked scores only).
  static constexpr int kEmuPairs = (D == 64) ? FA_FWD_EMU_PAIRS_D64 : FA_FWD_EMU_PAIRS_D128;
  static constexpr int kTileBytes = kBN * D * 2;   // one K or V tile (bf16)
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kColBlocks = D / 64;        // 128-byte column blocks per row
  static constexpr int kBlockBytes = 128 * 128;    // one column block of a 128-row tile
  static constexpr uint32_t kS0 = 0, kS1 = 128;
  static constexpr uint32_t kO0 = 256, kO1 = 256 + (D == 64 ? 64 : 128);
  static constexpr uint32_t kPOff = 64;            // P (bf16 pairs) inside S's columns
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = kOffQ + 2 * kQBytes;
  static constexpr int kOffEnd = kOffKV + kSlots * kTileBytes;
  static_assert(kSlots <= kMaxSlots, "ring barriers");
};

// Ring position of the n-th K/V tile loaded (K_j is n = 2j, V_j is n = 2j + 1).
template <int kSlots>
__device__ __forceinline__ int ring_slot(int n) { return n % kSlots; }
template <int kSlots>
__device__ __forceinline__ uint32_t ring_phase(int n) { return (n / kSlots) & 1; }

struct alignas(16) CtlCore {
  uint64_t q_full;
  uint64_t kv_full[kMaxSlots], kv_empty[kMaxSlots];
  uint64_t s_full[2], p_half[2], p_full[2];
  uint64_t o_ready[2];       // query tile t's last P V has completed
  uint64_t o_done;
  uint64_t never;            // signalled by nothing (wait-limit test hook)
  uint64_t qt_full[2], qt_empty[2];   // per query tile Q buffer (persistent form)
  uint64_t item_full[4], item_empty[4];   // work-item ring (persistent form)
  int item_id[4];
  uint32_t tmem_base;
  int abort;
  int skip;                  // the error word was set at launch: the CTA does nothing
  int ntiles;
  int nlive[2];              // key tiles query tile t sees (skipping form)
};

// Key-tile lists of the skipping form. The lockstep form walks key tiles
// 0 .. T-1 and needs none.
struct TileLists {
  uint16_t tiles[kMaxTiles];
  uint8_t dead[kMaxTiles];       // bit t: query tile t sees nothing of this key tile
  uint16_t seen[kMaxTiles][2];   // [n][t]: n-th key tile query tile t sees, | kFullBit
};

// Flag on a list entry: every (query, key) pair of the tile is visible, so
// its scores need no masking.
constexpr uint16_t kFullBit = 0x8000;

template <bool kSkip>
struct Ctl : CtlCore {};
template <>
struct Ctl<true> : CtlCore {
  TileLists l;
};

struct FwdParams {
  CUtensorMap tq, tk, tv;    // [B*H][N][d] bf16, box {64, 128, 1}, 128B swizzle
  CUtensorMap to;            // O, the same layout (dense batches: TMA-stored epilogue)
  __nv_bfloat16* O;
  float* LSE;
  const uint8_t* mask;
  unsigned* err;
  int N, Hq, Hkv, nb, nblk, causal, BH;
  MaskMod mod;               // keys each query sees (the causal flag is its wr = 0)
  float c;                   // scale * log2(e)
  float cap1, cap2;          // soft-capping: scores in log2 units = cap1 * tanh(cap2 * q.k)
  const int* cu;             // variable-length batch: sequence offsets [B+1], or null
  int total;                 // packed rows (variable-length batch)
  int chunk;                 // heads interleaved in launch order
  long long stall;           // > 0: injected wait of this many cycles (test hook)
};

// 32 pairs of scores -> p = 2^(s*c - mu) packed to bf16 pairs, with the
// fp32 values added into four pair accumulators. With kEmu, kEmuPairs of
// every 8 pairs use the FMA-pipe exp2 (finite inputs only), the rest MUFU.
template <bool kEmu, int kEmuPairs>
__device__ __forceinline__ void exp_pack32(const uint32_t* sr, float2 c2, float2 nmu2,
                                           float2 (&acc)[4], uint32_t (&pk)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float2 x =
        ffma2(make_float2(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), c2, nmu2);
    float2 e;
    if (kEmu && (i & 7) < kEmuPairs)
      e = exp2_poly2(x);
    else
      e = make_float2(ex2(x.x), ex2(x.y));
    acc[i & 3] = fadd2(acc[i & 3], e);
    pk[i] = pack_bf16(e.x, e.y);
  }
}

// The online-softmax step of one key tile for this thread's row, after its
// scores sr (already masked: -inf where not visible; in log2 units once
// multiplied by c) have been loaded from TMEM: row maximum, a move of the
// reference maximum m_ref when the tile's maximum exceeds it by more than
// kTau (l and, for n > 0, the TMEM accumulator rescaled by
// alpha = 2^(m_old - m_new)), p = 2^(s*c - m_ref) into the P columns of S
// (half a row at a time: p_half after the first 64 keys so P V can start,
// p_full after all of them) and l += rowsum p. n is the tile's index within
// the item (no accumulator to rescale before the first).
template <int D, int kEmuPairs>
__device__ __forceinline__ void softmax_tile(uint32_t (&sr)[128], bool need_mask, float c, int n,
                                             float& m_ref, float& l, uint32_t sreg,
                                             uint32_t preg, uint32_t oreg, uint64_t* p_half,
                                             uint64_t* p_full, int lane) {
  // Row maximum: eight independent chains of three-input max.
  float m8[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float* v = reinterpret_cast<const float*>(&sr[16 * k]);
    float m = fmax3(v[0], v[1], v[2]);
#pragma unroll
    for (int i = 3; i < 15; i += 2) m = fmax3(m, v[i], v[i + 1]);
    m8[k] = fmaxf(m, v[15]);
  }
  const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]),
                         fmaxf(m8[6], m8[7]));
  const float mx2 = mx * c;
  const bool grow = mx2 > m_ref + kTau;
  float alpha = 1.f;
  if (grow) {
    alpha = ex2(m_ref - mx2);   // 0 when there was no reference yet
    m_ref = mx2;
    l *= alpha;
  }
  const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
  // p = 2^(s*c - mu), two lanes per FMA, four pair accumulators for the
  // sum; P goes to TMEM half a row at a time to keep registers free. In
  // tiles without masked scores a share of the exponentials (kEmuPairs of
  // every 8 pairs) can run on the FMA pipe (exp2_poly2) instead of MUFU.
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
  const float2 c2 = make_float2(c, c), nmu2 = make_float2(-mu, -mu);
  // The MMA warp starts P V on the first 64 keys as soon as their P is in
  // TMEM (p_half), while this warpgroup computes the second half.
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    uint32_t pk[32];
    if (need_mask)
      exp_pack32<false, kEmuPairs>(&sr[64 * hf], c2, nmu2, acc, pk);
    else
      exp_pack32<true, kEmuPairs>(&sr[64 * hf], c2, nmu2, acc, pk);
    tmem_st32(preg + 32 * hf, pk);
    if (hf == 0) {
      // The accumulator holds P V of earlier tiles (complete: the commit
      // that signalled S_t came after them); rescale it where the
      // reference moved, before any P V of this tile is issued.
      if (__any_sync(0xffffffffu, grow && n > 0)) {
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(oreg + cc * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(oreg + cc * 32, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_half);
    }
  }
  const float2 a01 = fadd2(acc[0], acc[1]), a23 = fadd2(acc[2], acc[3]);
  l += (a01.x + a01.y) + (a23.x + a23.y);
  tmem_st_wait();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(p_full);
}

// Writes this thread's output row O = acc / l (bf16; zeros when no P V ran
// into the accumulator) into a 128-row tile staged in shared memory in the
// TMA's 128-byte-swizzled layout: 64-column block cb at cb * 16 KB, row r at
// r * 128 bytes, 16-byte chunk c of the row at ((c ^ (r & 7)) << 4). One TMA
// store per column block then writes whole lines of O.
template <int D>
__device__ __forceinline__ void stage_row(uint32_t oreg, bool have_o, float l, int r,
                                          uint8_t* stage) {
  const float inv = (l > 0.f) ? 1.f / l : 0.f;
  // the whole row in one TMEM round trip (the score registers are free here)
  uint32_t o[D];
  if (have_o) {
    if constexpr (D == 128)
      tmem_ld128(oreg, o);
    else
      tmem_ld64(oreg, o);
  } else {
#pragma unroll
    for (int i = 0; i < D; ++i) o[i] = 0u;
  }
#pragma unroll
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      w[i] = pack_bf16(__uint_as_float(o[32 * cc + 2 * i]) * inv,
                       __uint_as_float(o[32 * cc + 2 * i + 1]) * inv);
    uint8_t* rowp = stage + (cc >> 1) * 16384 + r * 128;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = 4 * (cc & 1) + q;
      *reinterpret_cast<uint4*>(rowp + ((c ^ (r & 7)) << 4)) =
          make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
    }
  }
}

// Stores this thread's output row: O = acc / l (bf16, 16-byte vectors) from
// the TMEM accumulator (or zeros when no P V ran into it) and LSE =
// (m_ref + log2 l) ln 2 (-inf for a row with no visible key).
template <int D>
__device__ __forceinline__ void store_row(uint32_t oreg, bool have_o, float m_ref, float l,
                                          bool valid, __nv_bfloat16* out, float* lse_out) {
  const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t o[32];
    if (have_o) {
      tmem_ld32(oreg + cc * 32, o);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = 0u;
    }
    uint4 v[4];
    uint32_t* vw = reinterpret_cast<uint32_t*>(v);
#pragma unroll
    for (int i = 0; i < 16; ++i)
      vw[i] = pack_bf16(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
    if (valid) {
      uint4* dst = reinterpret_cast<uint4*>(out + cc * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = v[i];
    }
  }
  if (valid) *lse_out = (l > 0.f) ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
}

// Bounded wait that ignores the abort flag (used only to drain in-flight work).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) break;
  }
}

template <int D, bool kVarlen, bool kSkip, bool kCap>
__global__ void __launch_bounds__(kThreads, 1) fwd_kernel(const __grid_constant__ FwdParams p) {
  using C = Cfg<D, kSkip>;
  constexpr int kSlots = C::kSlots;
  extern __shared__ uint8_t smem_raw[];
  Ctl<kSkip>& ctl = *reinterpret_cast<Ctl<kSkip>*>(smem_raw);
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t tile_addr = (raw_addr + sizeof(Ctl<kSkip>) + 1023u) & ~1023u;
  uint8_t* tiles_base = smem_raw + (tile_addr - raw_addr);

  // Heads are taken p.chunk at a time (their K/V stay in L2 during a wave);
  // inside a chunk the query blocks with the longest causal rows start first.
  int bh, rblk;
  chunked_order(blockIdx.x, p.nblk, p.BH, p.chunk, bh, rblk);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blk = p.nblk - 1 - rblk;
  const int h = bh % p.Hq, b = bh / p.Hq;
  const int bhk = b * p.Hkv + h / (p.Hq / p.Hkv);
  const int q0 = blk * 2 * kBM;
  const int qb0 = 2 * blk, qb1 = 2 * blk + 1;   // 128-row mask blocks of the two tiles
  // Dense: rows 0..N-1 of plane (b, h). Variable-length batch: sequence b is
  // rows cu[b] .. cu[b+1]-1 of the packed tensors (planes are heads); blocks
  // past its end have nothing to do. Offsets are clamped to [0, total].
  int N = p.N, nb = p.nb, row0 = 0, qplane = bh, kplane = bhk;
  if constexpr (kVarlen) {
    const int s0 = min(max(p.cu[b], 0), p.total);
    const int s1 = min(max(p.cu[b + 1], s0), p.total);
    N = min(s1 - s0, p.N);
    if (q0 >= N) return;
    nb = (N + kBN - 1) / kBN;
    row0 = s0;
    qplane = h;
    kplane = h / (p.Hq / p.Hkv);
  }
  // Key tiles either query tile can see end before kb_end. The lockstep form
  // runs without a block mask, a left window edge or documents, so every key
  // tile below kb_end is seen by one of the two query tiles: its list is
  // 0 .. kb_end-1 and needs no storage.
  const int kb_end = min(nb, mod_last_key(p.mod, qb1 * kBM + kBM - 1, N) / kBN + 1);

  // K/V ring loads issued before the block barrier below (lockstep form):
  // K_0 only, so the other threads do not wait long at the barrier for the
  // issuing thread
  const int pre_loads = kSkip ? 0 : 1;
  if (threadIdx.x == 0) {
    // A launch whose error word is already set (an earlier wait ran out and
    // nobody has read the word yet) does no work: its inputs may be invalid.
    // This one thread reads the word (while it sets up the barriers) and the
    // whole CTA leaves together after the block barrier below, before any
    // wait (another CTA may set the word meanwhile, so per-thread reads
    // could disagree).
    const unsigned err_word = *reinterpret_cast<volatile unsigned*>(p.err);
    mbar_init(&ctl.q_full, 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&ctl.kv_full[s], 1);
      mbar_init(&ctl.kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&ctl.s_full[t], 1);
      mbar_init(&ctl.p_half[t], 4);
      mbar_init(&ctl.p_full[t], 4);
      mbar_init(&ctl.o_ready[t], 1);
    }
    mbar_init(&ctl.o_done, 1);
    mbar_init(&ctl.never, 1);
    ctl.abort = 0;
    if constexpr (!kSkip) ctl.ntiles = kb_end;
    fence_mbar_init();
    {
      // This thread is also the TMA producer: the Q tiles and, in the
      // lockstep form, K_0 start now, so their latency (and that of the
      // error-word read) overlaps the TMEM allocation, the tile lists and the
      // block barrier. A CTA that then finds the word set waits for these
      // copies to land and does nothing else.
      prefetch_tmap(&p.tq);
      prefetch_tmap(&p.tk);
      prefetch_tmap(&p.tv);
      mbar_expect_tx(&ctl.q_full, 2 * C::kQBytes);
      for (int t = 0; t < 2; ++t)
        for (int cb = 0; cb < C::kColBlocks; ++cb)
          tma_load_3d(tiles_base + C::kOffQ + t * C::kQBytes + cb * C::kBlockBytes, &p.tq,
                      &ctl.q_full, cb * 64, row0 + q0 + t * kBM, qplane);
      for (int n = 0; n < pre_loads; ++n) {
        mbar_expect_tx(&ctl.kv_full[n], C::kTileBytes);
        for (int cb = 0; cb < C::kColBlocks; ++cb)
          tma_load_3d(tiles_base + C::kOffKV + n * C::kTileBytes + cb * C::kBlockBytes,
                      (n & 1) ? &p.tv : &p.tk, &ctl.kv_full[n], cb * 64, row0 + (n >> 1) * kBN,
                      kplane);
      }
    }
    ctl.skip = err_word != 0u;
  }
  if (warp == 2) {
    tmem_alloc(&ctl.tmem_base, 512);
    tmem_relinquish();
  }
  if constexpr (kSkip) {
    if (warp == 3) {
      // Key tiles either query tile can see, in increasing order, and each
      // query tile's own list (entries flagged kFullBit need no masking).
      int count = 0, live0 = 0, live1 = 0;
      for (int kb0 = 0; kb0 < kb_end; kb0 += 32) {
        const int kb = kb0 + lane;
        int k0 = kTileEmpty, k1 = kTileEmpty;
        if (kb < kb_end) {
          const int c0 = kb * kBN, c1 = c0 + kBN - 1;
          if (!p.mask || p.mask[(size_t)qb0 * p.nb + kb])
            k0 = mod_classify(p.mod, qb0 * kBM, qb0 * kBM + kBM - 1, c0, c1, N);
          if (qb1 < nb && (!p.mask || p.mask[(size_t)qb1 * p.nb + kb]))
            k1 = mod_classify(p.mod, qb1 * kBM, qb1 * kBM + kBM - 1, c0, c1, N);
        }
        const bool a0 = k0 != kTileEmpty, a1 = k1 != kTileEmpty;
        const bool act = a0 || a1;
        const unsigned below = (1u << lane) - 1u;
        const unsigned bal = __ballot_sync(0xffffffffu, act);
        if (act) {
          const int pos = count + __popc(bal & below);
          ctl.l.tiles[pos] = static_cast<uint16_t>(kb);
          ctl.l.dead[pos] = static_cast<uint8_t>((a0 ? 0 : 1) | (a1 ? 0 : 2));
        }
        const unsigned bal0 = __ballot_sync(0xffffffffu, a0);
        const unsigned bal1 = __ballot_sync(0xffffffffu, a1);
        if (a0)
          ctl.l.seen[live0 + __popc(bal0 & below)][0] =
              static_cast<uint16_t>(kb | (k0 == kTileFull ? kFullBit : 0));
        if (a1)
          ctl.l.seen[live1 + __popc(bal1 & below)][1] =
              static_cast<uint16_t>(kb | (k1 == kTileFull ? kFullBit : 0));
        live0 += __popc(bal0);
        live1 += __popc(bal1);
        count += __popc(bal);
      }
      if (lane == 0) {
        ctl.ntiles = count;
        ctl.nlive[0] = live0;
        ctl.nlive[1] = live1;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = ctl.tmem_base;
  if (ctl.skip) {   // the error word was set at launch: no work
    if (threadIdx.x == 0) {
      drain_wait(&ctl.q_full, 0);
      for (int n = 0; n < pre_loads; ++n) drain_wait(&ctl.kv_full[n], 0);
    }
    if (warp == 2) tmem_dealloc(tm, 512);
    return;
  }
  const int T = ctl.ntiles;
  const Guard g{&ctl.abort, p.err};
  // j-th key tile of the CTA's list
  auto tile_of = [&](int j) -> int {
    if constexpr (kSkip) return ctl.l.tiles[j];
    else return j;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // (Q and the first pre_loads ring tiles were issued before the block
      // barrier.) K_0, V_0, K_1, V_1, ... into the slot ring, each slot
      // reused once the MMA warp has released the tile kSlots loads earlier.
      int issued = pre_loads;
      for (int n = pre_loads; n < 2 * T; ++n) {
        const int s = ring_slot<kSlots>(n);
        if (n >= kSlots && !mbar_wait_ready_first(&ctl.kv_empty[s], ring_phase<kSlots>(n - kSlots), g)) break;
        const int kb = tile_of(n >> 1);
        const CUtensorMap* m = (n & 1) ? &p.tv : &p.tk;
        mbar_expect_tx(&ctl.kv_full[s], C::kTileBytes);
        for (int cb = 0; cb < C::kColBlocks; ++cb)
          tma_load_3d(tiles_base + C::kOffKV + s * C::kTileBytes + cb * C::kBlockBytes, m,
                      &ctl.kv_full[s], cb * 64, row0 + kb * kBN, kplane);
        issued = n + 1;
      }
      // Every issued copy has landed before the CTA may exit.
      drain_wait(&ctl.q_full, 0);
      for (int s = 0; s < kSlots && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / kSlots) * kSlots;   // last load into slot s
        drain_wait(&ctl.kv_full[s], ring_phase<kSlots>(last));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && T > 0) {
      constexpr uint32_t idS = idesc_bf16(kBM, kBN, false, false);
      constexpr uint32_t idO = idesc_bf16(kBM, D, false, true);
      // Base descriptors, built once: Q tile 0 (tile 1 follows it), ring slot
      // 0 read as a K tile (K-major) and as a V tile (MN-major); every MMA
      // operand below is one of them plus a byte offset (sdesc_at), which
      // keeps the issue path after each P signal short.
      const uint64_t dq0 = sdesc_sw128(smem_u32(tiles_base + C::kOffQ), 16, 1024);
      const uint64_t dk0 = sdesc_sw128(smem_u32(tiles_base + C::kOffKV), 16, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(tiles_base + C::kOffKV), C::kBlockBytes, 1024);
      auto wait_tile = [&](int n) {
        return mbar_wait_ready_first(&ctl.kv_full[ring_slot<kSlots>(n)], ring_phase<kSlots>(n), g);
      };
      auto release_tile = [&](int n) { mma_commit(&ctl.kv_empty[ring_slot<kSlots>(n)]); };
      // S_t = Q_t K_j^T
      auto issue_s = [&](int t, int j) {
        const uint64_t dq = sdesc_at(dq0, t * C::kQBytes);
        const uint64_t dk = sdesc_at(dk0, ring_slot<kSlots>(2 * j) * C::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBlockBytes + (kk & 3) * 32;
          mma_ss(tm + (t ? C::kS1 : C::kS0), sdesc_at(dq, off), sdesc_at(dk, off), idS, kk > 0);
        }
      };
      // O_t += P_t V_j over keys 64*hf .. 64*hf+63 of the tile.
      auto issue_pv = [&](int t, int j, bool acc, int hf) {
        const uint64_t dv = sdesc_at(dv0, ring_slot<kSlots>(2 * j + 1) * C::kTileBytes);
        const uint32_t pt = tm + (t ? C::kS1 : C::kS0) + C::kPOff;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int kk = 4 * hf + k4;
          mma_ts(tm + (t ? C::kO1 : C::kO0), pt + kk * 8, sdesc_at(dv, kk * 16 * 128), idO,
                 (acc || kk > 0));
        }
      };
      if constexpr (kSkip) {
        // A query tile skips the key tiles it sees nothing of (block mask,
        // causal diagonal, window edge): no Q K^T, softmax or P V for it there.
        // n0, n1 count the tiles each query tile has been through; its barriers
        // (s_full, p_half, p_full) complete once per such tile. The live bits
        // of a tile (bit t: query tile t sees it) are read one tile ahead, so
        // no shared-memory load sits between a signal and the next issue.
        const int nl0 = ctl.nlive[0], nl1 = ctl.nlive[1];
        int n0 = 0, n1 = 0;
        int live_next = T > 0 ? (~ctl.l.dead[0] & 3) : 0;
        bool ok = injected_stall(&ctl.never, p.stall, g) && mbar_wait_ready_first(&ctl.q_full, 0, g) &&
                  wait_tile(0);
        if (ok) {
          tc_fence_after();
          if (live_next & 1) {
            issue_s(0, 0);
            mma_commit(&ctl.s_full[0]);
          }
          if (live_next & 2) {
            issue_s(1, 0);
            mma_commit(&ctl.s_full[1]);
          }
          release_tile(0);
        }
        for (int j = 0; ok && j < T; ++j) {
          const bool more = j + 1 < T;
          const int live_cur = live_next;
          live_next = more ? (~ctl.l.dead[j + 1] & 3) : 0;
          if (!(ok = wait_tile(2 * j + 1))) break;
          if (live_cur & 1) {
            if (!(ok = mbar_wait_ready_first(&ctl.p_half[0], n0 & 1, g))) break;
            tc_fence_after();
            issue_pv(0, j, n0 > 0, 0);
            if (!(ok = mbar_wait_ready_first(&ctl.p_full[0], n0 & 1, g))) break;
            tc_fence_after();
            issue_pv(0, j, n0 > 0, 1);
            if (++n0 == nl0) mma_commit(&ctl.o_ready[0]);
          }
          if (more) {
            if (!(ok = wait_tile(2 * j + 2))) break;
            tc_fence_after();
            if (live_next & 1) {
              issue_s(0, j + 1);
              mma_commit(&ctl.s_full[0]);
            }
          }
          if (live_cur & 2) {
            if (!(ok = mbar_wait_ready_first(&ctl.p_half[1], n1 & 1, g))) break;
            tc_fence_after();
            issue_pv(1, j, n1 > 0, 0);
            if (!(ok = mbar_wait_ready_first(&ctl.p_full[1], n1 & 1, g))) break;
            tc_fence_after();
            issue_pv(1, j, n1 > 0, 1);
            if (++n1 == nl1) mma_commit(&ctl.o_ready[1]);
          }
          release_tile(2 * j + 1);   // V_j
          if (more) {
            if (live_next & 2) {
              issue_s(1, j + 1);
              mma_commit(&ctl.s_full[1]);
            }
            release_tile(2 * j + 2);   // K_{j+1}
          }
        }
        // Every query tile's epilogue gets its signal, also after an abort.
        if (n0 != nl0 || nl0 == 0) mma_commit(&ctl.o_ready[0]);
        if (n1 != nl1 || nl1 == 0) mma_commit(&ctl.o_ready[1]);
      } else {
        bool ok = injected_stall(&ctl.never, p.stall, g) && mbar_wait_ready_first(&ctl.q_full, 0, g) &&
                  wait_tile(0);
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
          mma_commit(&ctl.s_full[0]);
          issue_s(1, 0);
          mma_commit(&ctl.s_full[1]);
          release_tile(0);
        }
        for (int j = 0; ok && j < T; ++j) {
          const bool more = j + 1 < T;
          // V_j and K_{j+1} (long landed as a rule) are checked here, while P
          // is still being computed, so that nothing but the P signals sits
          // between a tile's last P V and its next S.
          if (!(ok = wait_tile(2 * j + 1) && (!more || wait_tile(2 * j + 2)) &&
                     mbar_wait_ready_first(&ctl.p_half[0], j & 1, g)))
            break;
          tc_fence_after();
          issue_pv(0, j, j > 0, 0);
          if (!(ok = mbar_wait_ready_first(&ctl.p_full[0], j & 1, g))) break;
          tc_fence_after();
          issue_pv(0, j, j > 0, 1);
          // the last P V of a query tile: its epilogue may start
          if (!more) mma_commit(&ctl.o_ready[0]);
          if (more) {
            issue_s(0, j + 1);
            mma_commit(&ctl.s_full[0]);
          }
          if (!(ok = mbar_wait_ready_first(&ctl.p_half[1], j & 1, g))) break;
          tc_fence_after();
          issue_pv(1, j, j > 0, 0);
          if (!(ok = mbar_wait_ready_first(&ctl.p_full[1], j & 1, g))) break;
          tc_fence_after();
          issue_pv(1, j, j > 0, 1);
          if (!more) mma_commit(&ctl.o_ready[1]);
          release_tile(2 * j + 1);   // V_j
          if (more) {
            issue_s(1, j + 1);
            mma_commit(&ctl.s_full[1]);
            release_tile(2 * j + 2);   // K_{j+1}
          }
        }
      }
      mma_commit(&ctl.o_done);
      drain_wait(&ctl.o_done, 0);   // no MMA may still run when TMEM is freed
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;           // query tile of this warpgroup
    const int wq = warp & 3;                 // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;            // row inside the tile
    const int row = q0 + t * kBM + r;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t sreg = tm + (t ? C::kS1 : C::kS0) + lane_off;
    const uint32_t oreg = tm + (t ? C::kO1 : C::kO0) + lane_off;
    // With soft-capping the scores are transformed into log2 units before the
    // softmax (score modifier first, then the mask), so the exponent scale is 1.
    const float c = kCap ? 1.f : p.c;
    const int tile_row0 = q0 + t * kBM;
    float m_ref = -INFINITY, l = 0.f;
    // Skipping form: the keys this row sees (before the block mask, which is
    // per tile), looked up once (documents take binary searches). The
    // lockstep form has no documents and no left edge: its bounds are cheap
    // to recompute where a tile needs masking.
    int row_lo = 0, row_hi = N - 1;
    if constexpr (kSkip) mod_row_keys(p.mod, row, N, row_lo, row_hi);
    // Lockstep form: every tile of the list, n = it. Skipping form: only the
    // tiles this query tile sees, it = 2n + t walking entry [n][t] of its list.
    constexpr int kStep = kSkip ? 2 : 1;
    const int it_end = kSkip ? 2 * ctl.nlive[t] + t : T;
    int it = kSkip ? t : 0;
    for (; it < it_end; it += kStep) {
      const int n = kSkip ? (it >> 1) : it;   // tiles of this query tile so far
      if (!mbar_wait_ready_first(&ctl.s_full[t], n & 1, g)) break;
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld128(sreg, sr);
      if constexpr (kCap) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          sr[i] = __float_as_uint(p.cap1 * tanh_ex2(__uint_as_float(sr[i]) * p.cap2));
      }
      int col0;
      bool dead = false, need_mask;
      if constexpr (kSkip) {
        const int e = (&ctl.l.seen[0][0])[it];
        col0 = (e & ~kFullBit) * kBN;
        need_mask = !(e & kFullBit);
      } else {
        // lockstep: key tile it; this query tile may see none of it (the
        // causal diagonal or a right window edge of the other tile, or a
        // second tile past the end of the sequence)
        col0 = it * kBN;
        // (the classification of mod_classify without documents or a left
        // edge, and keys past N masked whatever the rows)
        const int wr = p.mod.wr, pre1 = p.mod.prefix - 1;
        dead = (t == 1 && qb1 >= nb) || (wr >= 0 && col0 > max(tile_row0 + kBM - 1 + wr, pre1));
        need_mask = dead || col0 + kBN > N || (wr >= 0 && col0 + kBN - 1 > max(tile_row0 + wr, pre1));
      }
      if (need_mask) {
        if constexpr (!kSkip) mod_row_keys(p.mod, row, N, row_lo, row_hi);
        // this row's visible columns of the tile: [lo, hi] relative to col0
        const int lo = row_lo - col0;
        const int hi = dead ? lo - 1 : row_hi - col0;
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i < lo || i > hi) sr[i] = __float_as_uint(-INFINITY);
      }
      softmax_tile<D, C::kEmuPairs>(sr, need_mask, c, n, m_ref, l, sreg, sreg + C::kPOff, oreg,
                                    &ctl.p_half[t], &ctl.p_full[t], lane);
    }
    // ------------------------------------------------------------ epilogue
    // The accumulator holds something only if some P V ran into it.
    bool have_o;
    if constexpr (kSkip)
      have_o = __any_sync(0xffffffffu, it > 1);
    else
      have_o = T > 0;
    if (have_o) {
      // this query tile's last P V has completed (its S MMAs, which read the
      // Q buffer, came before it)
      mbar_wait_ready_first(&ctl.o_ready[t], 0, g);
      tc_fence_after();
    } else {
      // no MMA read this tile's Q buffer, but its load may still be landing:
      // wait for it before the buffer is reused for the output
      mbar_wait_ready_first(&ctl.q_full, 0, g);
    }
    const bool valid = row < N;
    if constexpr (!kVarlen) {
      // O through the free Q buffer of this tile and TMA stores (rows at or
      // past N are clipped by the tensor map); LSE row by row
      uint8_t* stage = tiles_base + C::kOffQ + t * C::kQBytes;
      stage_row<D>(oreg, have_o, l, r, stage);
      if (valid)
        p.LSE[(size_t)bh * p.N + row] = (l > 0.f) ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
      fence_async_smem();
      named_sync(1 + t, 128);
      if (warp == 4 + 4 * t && lane == 0) {
#pragma unroll
        for (int cb = 0; cb < C::kColBlocks; ++cb)
          tma_store_3d(&p.to, stage + cb * C::kBlockBytes, cb * 64, tile_row0, bh);
        bulk_commit();
        bulk_wait_read0();   // the staging buffer is read before the CTA exits
      }
    } else {
      // packed batch: a 128-row box could reach into the next sequence, so
      // rows are stored one by one ([total][H][d])
      const size_t o_base = ((size_t)row0 * p.Hq + h) * D;
      const size_t lse_base = (size_t)h * p.total + row0;
      store_row<D>(oreg, have_o, m_ref, l, valid,
                   p.O + o_base + (size_t)(valid ? row : 0) * p.Hq * D,
                   p.LSE + lse_base + (valid ? row : 0));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

// Persistent form of the lockstep forward (dense and causal launches without
// a block mask, left window edge or documents): one CTA per SM takes work
// items (a (batch, head) and a block of two 128-row query tiles, numbered in
// the launch order of the one-item form) from a queue, so what a CTA of the
// one-item form pays per item -- set-up, the first S waiting for Q, the
// epilogue with the tensor core idle, the gap before the next CTA starts --
// is paid once per SM or overlapped:
//  * the producer draws item numbers from a counter in the workspace's
//    error block (atomicAdd), which balances causal items of different
//    lengths, and hands them to the MMA and softmax warps through a ring of
//    kItemRing entries; the last CTA to leave resets the counter;
//  * the Q tile t of the next item is loaded as soon as the last S_t of the
//    current one has read the buffer, and the K/V ring runs on across items;
//  * the epilogue stages O in a buffer of its own and writes it with TMA
//    stores, so the next item's Q is not disturbed.
// Barrier phases count tiles and items per CTA; each item's softmax state
// starts afresh.
constexpr int kItemRing = 4;

template <int D>
struct PCfg {
  static constexpr int kSlots = (D == 64) ? 8 : 3;   // K/V ring (3 measured as fast as 5)
  static constexpr int kTileBytes = kBN * D * 2;
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kColBlocks = D / 64;
  static constexpr int kBlockBytes = 128 * 128;
  static constexpr int kEmuPairs = Cfg<D, false>::kEmuPairs;
  static constexpr uint32_t kS0 = 0, kS1 = 128;
  static constexpr uint32_t kO0 = 256, kO1 = 256 + (D == 64 ? 64 : 128);
  static constexpr uint32_t kPOff = 64;
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kQBytes;
  static constexpr int kOffStage = kOffKV + kSlots * kTileBytes;   // O staging, two tiles
  static constexpr int kOffEnd = kOffStage + 2 * kQBytes;
  static_assert(kSlots <= kMaxSlots, "ring barriers");
};

template <int D, bool kCap>
__global__ void __launch_bounds__(kThreads, 1) fwd_persist_kernel(const __grid_constant__ FwdParams p) {
  using C = PCfg<D>;
  constexpr int kSlots = C::kSlots;
  extern __shared__ uint8_t smem_raw[];
  Ctl<false>& ctl = *reinterpret_cast<Ctl<false>*>(smem_raw);
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t tile_addr = (raw_addr + sizeof(Ctl<false>) + 1023u) & ~1023u;
  uint8_t* tiles_base = smem_raw + (tile_addr - raw_addr);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int W = p.BH * p.nblk;   // work items
  const int N = p.N, nb = p.nb;
  unsigned* const next_item = p.err + 16;   // queue counter (workspace byte 64)
  unsigned* const ctas_done = p.err + 17;   // CTAs that have left (byte 68)

  // item w -> (bh, first query row, number of key tiles, kv plane)
  struct Item {
    int bh, q0, T, kplane;
  };
  auto item_of = [&](int w) {
    int bh, rblk;
    chunked_order(w, p.nblk, p.BH, p.chunk, bh, rblk);
    const int blk = p.nblk - 1 - rblk;
    Item it;
    it.bh = bh;
    it.q0 = blk * 2 * kBM;
    it.T = min(nb, mod_last_key(p.mod, (2 * blk + 1) * kBM + kBM - 1, N) / kBN + 1);
    it.kplane = (bh / p.Hq) * p.Hkv + (bh % p.Hq) / (p.Hq / p.Hkv);
    return it;
  };

  if (threadIdx.x == 0) {
    // a launch whose error word is already set does no work (see fwd_kernel)
    const unsigned err_word = *reinterpret_cast<volatile unsigned*>(p.err);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&ctl.kv_full[s], 1);
      mbar_init(&ctl.kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&ctl.qt_full[t], 1);
      mbar_init(&ctl.qt_empty[t], 1);
      mbar_init(&ctl.s_full[t], 1);
      mbar_init(&ctl.p_half[t], 4);
      mbar_init(&ctl.p_full[t], 4);
      mbar_init(&ctl.o_ready[t], 1);
    }
    for (int i = 0; i < kItemRing; ++i) {
      mbar_init(&ctl.item_full[i], 1);
      mbar_init(&ctl.item_empty[i], 9);   // the MMA thread and the eight softmax warps
    }
    mbar_init(&ctl.o_done, 1);
    mbar_init(&ctl.never, 1);
    ctl.abort = 0;
    fence_mbar_init();
    ctl.skip = err_word != 0u;
  }
  if (warp == 2) {
    tmem_alloc(&ctl.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = ctl.tmem_base;
  const Guard g{&ctl.abort, p.err};

  if (ctl.skip) {
    // no work
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer + queue
    if (lane == 0) {
      prefetch_tmap(&p.tq);
      prefetch_tmap(&p.tk);
      prefetch_tmap(&p.tv);
      prefetch_tmap(&p.to);
      int n = 0;              // K/V tiles loaded into the ring so far
      int qi[2] = {0, 0};     // loads of each Q tile buffer so far
      bool ok = true;
      for (int k = 0; ok; ++k) {
        // the next item for this CTA (or -1: the queue is empty)
        const int slot = k % kItemRing;
        if (k >= kItemRing &&
            !(ok = mbar_wait_ready_first(&ctl.item_empty[slot], ((k / kItemRing) - 1) & 1, g)))
          break;
        const unsigned w = atomicAdd(next_item, 1u);
        const int wi = (w < (unsigned)W) ? (int)w : -1;
        ctl.item_id[slot] = wi;
        mbar_arrive(&ctl.item_full[slot]);
        if (wi < 0) break;
        const Item it = item_of(wi);
        // Q tile t once the previous item's last S_t has read the buffer
        for (int t = 0; ok && t < 2; ++t) {
          if (qi[t] > 0 && !(ok = mbar_wait_ready_first(&ctl.qt_empty[t], (qi[t] - 1) & 1, g))) break;
          mbar_expect_tx(&ctl.qt_full[t], C::kQBytes);
          for (int cb = 0; cb < C::kColBlocks; ++cb)
            tma_load_3d(tiles_base + C::kOffQ + t * C::kQBytes + cb * C::kBlockBytes, &p.tq,
                        &ctl.qt_full[t], cb * 64, it.q0 + t * kBM, it.bh);
          ++qi[t];
        }
        for (int j = 0; ok && j < 2 * it.T; ++j, ++n) {
          const int s = ring_slot<kSlots>(n);
          if (n >= kSlots && !(ok = mbar_wait_ready_first(&ctl.kv_empty[s], ring_phase<kSlots>(n - kSlots), g)))
            break;
          mbar_expect_tx(&ctl.kv_full[s], C::kTileBytes);
          for (int cb = 0; cb < C::kColBlocks; ++cb)
            tma_load_3d(tiles_base + C::kOffKV + s * C::kTileBytes + cb * C::kBlockBytes,
                        (j & 1) ? &p.tv : &p.tk, &ctl.kv_full[s], cb * 64, (j >> 1) * kBN,
                        it.kplane);
        }
      }
      // Every issued copy has landed before the CTA may exit.
      for (int t = 0; t < 2; ++t)
        if (qi[t] > 0) drain_wait(&ctl.qt_full[t], (qi[t] - 1) & 1);
      for (int s = 0; s < kSlots && s < n; ++s) {
        const int last = s + ((n - 1 - s) / kSlots) * kSlots;
        drain_wait(&ctl.kv_full[s], ring_phase<kSlots>(last));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kBM, kBN, false, false);
      constexpr uint32_t idO = idesc_bf16(kBM, D, false, true);
      // base descriptors, as in the one-item form
      const uint64_t dq0 = sdesc_sw128(smem_u32(tiles_base + C::kOffQ), 16, 1024);
      const uint64_t dk0 = sdesc_sw128(smem_u32(tiles_base + C::kOffKV), 16, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(tiles_base + C::kOffKV), C::kBlockBytes, 1024);
      auto wait_tile = [&](int n) {
        return mbar_wait_ready_first(&ctl.kv_full[ring_slot<kSlots>(n)], ring_phase<kSlots>(n), g);
      };
      auto release_tile = [&](int n) { mma_commit(&ctl.kv_empty[ring_slot<kSlots>(n)]); };
      // S_t = Q_t K^T with K the ring tile n
      auto issue_s = [&](int t, int n) {
        const uint64_t dq = sdesc_at(dq0, t * C::kQBytes);
        const uint64_t dk = sdesc_at(dk0, ring_slot<kSlots>(n) * C::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBlockBytes + (kk & 3) * 32;
          mma_ss(tm + (t ? C::kS1 : C::kS0), sdesc_at(dq, off), sdesc_at(dk, off), idS, kk > 0);
        }
      };
      // O_t += P_t V over keys 64*hf .. 64*hf+63 of the ring tile n (a V tile)
      auto issue_pv = [&](int t, int n, bool acc, int hf) {
        const uint64_t dv = sdesc_at(dv0, ring_slot<kSlots>(n) * C::kTileBytes);
        const uint32_t pt = tm + (t ? C::kS1 : C::kS0) + C::kPOff;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int kk = 4 * hf + k4;
          mma_ts(tm + (t ? C::kO1 : C::kO0), pt + kk * 8, sdesc_at(dv, kk * 16 * 128), idO,
                 (acc || kk > 0));
        }
      };
      bool ok = injected_stall(&ctl.never, p.stall, g);
      int n = 0, nt = 0;   // ring tiles and softmax tiles so far
      for (int k = 0; ok; ++k) {
        const int slot = k % kItemRing;
        if (!(ok = mbar_wait_ready_first(&ctl.item_full[slot], (k / kItemRing) & 1, g))) break;
        const int wi = ctl.item_id[slot];
        mbar_arrive(&ctl.item_empty[slot]);
        if (wi < 0) break;
        const int T = item_of(wi).T;
        // K_j is ring tile n + 2j, V_j is n + 2j + 1
        for (int t = 0; t < 2; ++t) {
          if (!(ok = mbar_wait_ready_first(&ctl.qt_full[t], k & 1, g) && wait_tile(n))) break;
          tc_fence_after();
          issue_s(t, n);
          mma_commit(&ctl.s_full[t]);
          if (T == 1) mma_commit(&ctl.qt_empty[t]);
        }
        if (!ok) break;
        release_tile(n);
        for (int j = 0; ok && j < T; ++j) {
          const uint32_t ph = (nt + j) & 1;
          const bool more = j + 1 < T;
          // (as in the one-item form: the next K tile is checked before P)
          if (!(ok = wait_tile(n + 2 * j + 1) && (!more || wait_tile(n + 2 * j + 2)) &&
                     mbar_wait_ready_first(&ctl.p_half[0], ph, g)))
            break;
          tc_fence_after();
          issue_pv(0, n + 2 * j + 1, j > 0, 0);
          if (!(ok = mbar_wait_ready_first(&ctl.p_full[0], ph, g))) break;
          tc_fence_after();
          issue_pv(0, n + 2 * j + 1, j > 0, 1);
          if (!more) mma_commit(&ctl.o_ready[0]);
          if (more) {
            issue_s(0, n + 2 * j + 2);
            mma_commit(&ctl.s_full[0]);
            if (j + 2 == T) mma_commit(&ctl.qt_empty[0]);
          }
          if (!(ok = mbar_wait_ready_first(&ctl.p_half[1], ph, g))) break;
          tc_fence_after();
          issue_pv(1, n + 2 * j + 1, j > 0, 0);
          if (!(ok = mbar_wait_ready_first(&ctl.p_full[1], ph, g))) break;
          tc_fence_after();
          issue_pv(1, n + 2 * j + 1, j > 0, 1);
          if (!more) mma_commit(&ctl.o_ready[1]);
          release_tile(n + 2 * j + 1);   // V_j
          if (more) {
            issue_s(1, n + 2 * j + 2);
            mma_commit(&ctl.s_full[1]);
            if (j + 2 == T) mma_commit(&ctl.qt_empty[1]);
            release_tile(n + 2 * j + 2);   // K_{j+1}
          }
        }
        n += 2 * T;
        nt += T;
      }
      mma_commit(&ctl.o_done);
      drain_wait(&ctl.o_done, 0);   // no MMA may still run when TMEM is freed
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int t = (warp - 4) >> 2;           // query tile of this warpgroup
    const int wq = warp & 3;                 // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;            // row inside the tile
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t sreg = tm + (t ? C::kS1 : C::kS0) + lane_off;
    const uint32_t oreg = tm + (t ? C::kO1 : C::kO0) + lane_off;
    const float c = kCap ? 1.f : p.c;
    bool ok = true;
    int nt = 0;
    for (int k = 0; ok; ++k) {
      const int slot = k % kItemRing;
      if (!(ok = mbar_wait_ready_first(&ctl.item_full[slot], (k / kItemRing) & 1, g))) break;
      const int wi = ctl.item_id[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.item_empty[slot]);
      if (wi < 0) break;
      // (only what the tile loop needs stays live across it; the epilogue
      // decodes the item again)
      int tile_row0, T;
      {
        const Item it = item_of(wi);
        tile_row0 = it.q0 + t * kBM;
        T = it.T;
      }
      float m_ref = -INFINITY, l = 0.f;
      for (int j = 0; j < T; ++j) {
        if (!(ok = mbar_wait_ready_first(&ctl.s_full[t], (nt + j) & 1, g))) break;
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld128(sreg, sr);
        if constexpr (kCap) {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            sr[i] = __float_as_uint(p.cap1 * tanh_ex2(__uint_as_float(sr[i]) * p.cap2));
        }
        const int col0 = j * kBN;
        // as in the lockstep form: this query tile may see none of key tile j
        // (the second tile may also lie past the end of the sequence)
        const int wr = p.mod.wr, pre1 = p.mod.prefix - 1;
        const bool dead =
            tile_row0 >= N || (wr >= 0 && col0 > max(tile_row0 + kBM - 1 + wr, pre1));
        const bool need_mask =
            dead || col0 + kBN > N || (wr >= 0 && col0 + kBN - 1 > max(tile_row0 + wr, pre1));
        if (need_mask) {
          int row_lo, row_hi;
          mod_row_keys(p.mod, tile_row0 + r, N, row_lo, row_hi);
          const int lo = row_lo - col0;
          const int hi = dead ? lo - 1 : row_hi - col0;
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i < lo || i > hi) sr[i] = __float_as_uint(-INFINITY);
        }
        softmax_tile<D, C::kEmuPairs>(sr, need_mask, c, j, m_ref, l, sreg, sreg + C::kPOff, oreg,
                                      &ctl.p_half[t], &ctl.p_full[t], lane);
      }
      if (!ok) break;
      nt += T;
      // epilogue of this item: the last P V of this query tile has completed
      if (!(ok = mbar_wait_ready_first(&ctl.o_ready[t], k & 1, g))) break;
      tc_fence_after();
      const bool issuer = (warp == 4 + 4 * t) && lane == 0;   // of this tile's TMA stores
      uint8_t* stage = tiles_base + C::kOffStage + t * C::kQBytes;
      const int bh = item_of(wi).bh, row = tile_row0 + r;
      if (issuer) bulk_wait_read0();   // the previous item's store has read the staging
      named_sync(1 + t, 128);
      stage_row<D>(oreg, true, l, r, stage);
      if (row < N) p.LSE[(size_t)bh * N + row] = (l > 0.f) ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
      fence_async_smem();
      named_sync(1 + t, 128);
      if (issuer) {
#pragma unroll
        for (int cb = 0; cb < C::kColBlocks; ++cb)
          tma_store_3d(&p.to, stage + cb * C::kBlockBytes, cb * 64, tile_row0, bh);
        bulk_commit();
      }
    }
    if ((warp == 4 + 4 * t) && lane == 0) bulk_wait_read0();   // staging read before exit
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
  // The last CTA to leave resets the queue for the next launch (every CTA
  // has stopped drawing from it by now).
  if (threadIdx.x == 0 && atomicAdd(ctas_done, 1u) == gridDim.x - 1) {
    atomicExch(next_item, 0u);
    atomicExch(ctas_done, 0u);
  }
}

// Split form, for block-sparse launches: one 128-row query tile per CTA,
// whose visible key tiles (its list L, in increasing order) are dealt to the
// two softmax warpgroups in turn: stream 0 takes L[0], L[2], ..., stream 1
// L[1], L[3], .... Both streams read the one Q tile; each keeps its own
// online-softmax state and accumulator (O0 / O1 in TMEM), and the epilogue
// merges the two row by row (all in log2 units):
//   m = max(m0, m1), l = 2^(m0 - m) l0 + 2^(m1 - m) l1,
//   O = (2^(m0 - m) O0 + 2^(m1 - m) O1) / l.
// With a random block mask, two neighbouring query tiles seldom see the same
// key tile, so the paired skipping form runs most of its iterations with one
// live query tile; here both streams have a key tile in every iteration but
// the last. The K/V ring holds L's tiles in list order (K then V of each),
// each used by one stream only.
template <int D>
struct SCfg {
  static constexpr int kSlots = (D == 64) ? 10 : 5;
  static constexpr int kTileBytes = kBN * D * 2;
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kColBlocks = D / 64;
  static constexpr int kBlockBytes = 128 * 128;
  static constexpr int kEmuPairs = Cfg<D, false>::kEmuPairs;
  static constexpr uint32_t kS0 = 0, kS1 = 128;
  static constexpr uint32_t kO0 = 256, kO1 = 256 + (D == 64 ? 64 : 128);
  static constexpr uint32_t kPOff = 64;
  static constexpr int kOffQ = 0;                  // also the O staging in the epilogue
  static constexpr int kOffKV = kQBytes;
  static constexpr int kOffEnd = kOffKV + kSlots * kTileBytes;
  static_assert(kSlots <= kMaxSlots, "ring barriers");
};

struct CtlSplit : CtlCore {
  uint16_t tiles[kMaxTiles];   // L: visible key tiles of the query tile, | kFullBit
  float2 stat[2][kBM];         // per stream and row: (reference maximum, sum), log2 units
};

template <int D, bool kCap>
__global__ void __launch_bounds__(kThreads, 1) fwd_split_kernel(const __grid_constant__ FwdParams p) {
  using C = SCfg<D>;
  constexpr int kSlots = C::kSlots;
  extern __shared__ uint8_t smem_raw[];
  CtlSplit& ctl = *reinterpret_cast<CtlSplit*>(smem_raw);
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t tile_addr = (raw_addr + sizeof(CtlSplit) + 1023u) & ~1023u;
  uint8_t* tiles_base = smem_raw + (tile_addr - raw_addr);

  // one query tile per CTA: heads p.chunk at a time, tiles from the last
  int bh, rqb;
  chunked_order(blockIdx.x, p.nb, p.BH, p.chunk, bh, rqb);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = p.nb - 1 - rqb;
  const int h = bh % p.Hq, b = bh / p.Hq;
  const int bhk = b * p.Hkv + h / (p.Hq / p.Hkv);
  const int N = p.N, nb = p.nb;
  const int q0 = qb * kBM;
  const int kb_end = min(nb, mod_last_key(p.mod, q0 + kBM - 1, N) / kBN + 1);

  if (threadIdx.x == 0) {
    // (as in fwd_kernel: the error word is read once, and the CTA leaves
    // together after the block barrier if it was set)
    const unsigned err_word = *reinterpret_cast<volatile unsigned*>(p.err);
    mbar_init(&ctl.q_full, 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&ctl.kv_full[s], 1);
      mbar_init(&ctl.kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&ctl.s_full[t], 1);
      mbar_init(&ctl.p_half[t], 4);
      mbar_init(&ctl.p_full[t], 4);
      mbar_init(&ctl.o_ready[t], 1);
    }
    mbar_init(&ctl.o_done, 1);
    mbar_init(&ctl.never, 1);
    ctl.abort = 0;
    fence_mbar_init();
    prefetch_tmap(&p.tq);
    prefetch_tmap(&p.tk);
    prefetch_tmap(&p.tv);
    mbar_expect_tx(&ctl.q_full, C::kQBytes);
    for (int cb = 0; cb < C::kColBlocks; ++cb)
      tma_load_3d(tiles_base + C::kOffQ + cb * C::kBlockBytes, &p.tq, &ctl.q_full, cb * 64, q0,
                  bh);
    ctl.skip = err_word != 0u;
  }
  if (warp == 2) {
    tmem_alloc(&ctl.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 3) {
    // L: the key tiles below kb_end this query tile sees (block mask, then
    // the modifier's classification), flagged when wholly visible
    int count = 0;
    for (int kb0 = 0; kb0 < kb_end; kb0 += 32) {
      const int kb = kb0 + lane;
      int cls = kTileEmpty;
      if (kb < kb_end && (!p.mask || p.mask[(size_t)qb * nb + kb]))
        cls = mod_classify(p.mod, q0, q0 + kBM - 1, kb * kBN, kb * kBN + kBN - 1, N);
      const bool act = cls != kTileEmpty;
      const unsigned bal = __ballot_sync(0xffffffffu, act);
      if (act)
        ctl.tiles[count + __popc(bal & ((1u << lane) - 1u))] =
            static_cast<uint16_t>(kb | (cls == kTileFull ? kFullBit : 0));
      count += __popc(bal);
    }
    if (lane == 0) ctl.ntiles = count;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = ctl.tmem_base;
  if (ctl.skip) {
    if (threadIdx.x == 0) drain_wait(&ctl.q_full, 0);
    if (warp == 2) tmem_dealloc(tm, 512);
    return;
  }
  const int T = ctl.ntiles;                  // |L|
  const int T0 = (T + 1) / 2, T1 = T / 2;    // tiles of stream 0 and stream 1
  const Guard g{&ctl.abort, p.err};
  // list entry i (stream i & 1, its step i >> 1) is ring tiles 2i (K) and 2i + 1 (V)
  auto key_tile = [&](int i) { return static_cast<int>(ctl.tiles[i] & ~kFullBit); };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int n = 0; n < 2 * T; ++n) {
        const int s = ring_slot<kSlots>(n);
        if (n >= kSlots &&
            !mbar_wait_ready_first(&ctl.kv_empty[s], ring_phase<kSlots>(n - kSlots), g))
          break;
        mbar_expect_tx(&ctl.kv_full[s], C::kTileBytes);
        for (int cb = 0; cb < C::kColBlocks; ++cb)
          tma_load_3d(tiles_base + C::kOffKV + s * C::kTileBytes + cb * C::kBlockBytes,
                      (n & 1) ? &p.tv : &p.tk, &ctl.kv_full[s], cb * 64, key_tile(n >> 1) * kBN,
                      bhk);
        issued = n + 1;
      }
      drain_wait(&ctl.q_full, 0);
      for (int s = 0; s < kSlots && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / kSlots) * kSlots;
        drain_wait(&ctl.kv_full[s], ring_phase<kSlots>(last));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && T > 0) {
      constexpr uint32_t idS = idesc_bf16(kBM, kBN, false, false);
      constexpr uint32_t idO = idesc_bf16(kBM, D, false, true);
      const uint64_t dq = sdesc_sw128(smem_u32(tiles_base + C::kOffQ), 16, 1024);
      const uint64_t dk0 = sdesc_sw128(smem_u32(tiles_base + C::kOffKV), 16, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(tiles_base + C::kOffKV), C::kBlockBytes, 1024);
      auto wait_tile = [&](int n) {
        return mbar_wait_ready_first(&ctl.kv_full[ring_slot<kSlots>(n)], ring_phase<kSlots>(n), g);
      };
      auto release_tile = [&](int n) { mma_commit(&ctl.kv_empty[ring_slot<kSlots>(n)]); };
      // S_t = Q K^T for list entry i (stream t = i & 1), K the ring tile 2i
      auto issue_s = [&](int i) {
        const int t = i & 1;
        const uint64_t dk = sdesc_at(dk0, ring_slot<kSlots>(2 * i) * C::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBlockBytes + (kk & 3) * 32;
          mma_ss(tm + (t ? C::kS1 : C::kS0), sdesc_at(dq, off), sdesc_at(dk, off), idS, kk > 0);
        }
      };
      // O_t += P_t V over keys 64*hf .. 64*hf+63, V the ring tile 2i + 1
      auto issue_pv = [&](int i, bool acc, int hf) {
        const int t = i & 1;
        const uint64_t dv = sdesc_at(dv0, ring_slot<kSlots>(2 * i + 1) * C::kTileBytes);
        const uint32_t pt = tm + (t ? C::kS1 : C::kS0) + C::kPOff;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int kk = 4 * hf + k4;
          mma_ts(tm + (t ? C::kO1 : C::kO0), pt + kk * 8, sdesc_at(dv, kk * 16 * 128), idO,
                 (acc || kk > 0));
        }
      };
      bool ok = injected_stall(&ctl.never, p.stall, g) && mbar_wait_ready_first(&ctl.q_full, 0, g);
      // the first S of each stream
      for (int i = 0; ok && i < 2 && i < T; ++i) {
        if (!(ok = wait_tile(2 * i))) break;
        tc_fence_after();
        issue_s(i);
        mma_commit(&ctl.s_full[i]);
        release_tile(2 * i);   // K of entry i
      }
      // step j: entry 2j of stream 0, entry 2j + 1 of stream 1 (if any)
      for (int j = 0; ok && j < T0; ++j) {
        for (int t = 0; t < 2; ++t) {
          const int i = 2 * j + t;
          if (i >= T) break;
          const int nxt = i + 2;   // the stream's next entry
          if (!(ok = wait_tile(2 * i + 1) && mbar_wait_ready_first(&ctl.p_half[t], j & 1, g)))
            break;
          tc_fence_after();
          issue_pv(i, j > 0, 0);
          if (!(ok = mbar_wait_ready_first(&ctl.p_full[t], j & 1, g))) break;
          tc_fence_after();
          issue_pv(i, j > 0, 1);
          release_tile(2 * i + 1);   // V of entry i
          if (nxt < T) {
            // (its K is checked only now: with few ring slots it may still be
            // loading, and stream 1's P V must not wait for it)
            if (!(ok = wait_tile(2 * nxt))) break;
            tc_fence_after();
            issue_s(nxt);            // after P V in order: S overwrites P
            mma_commit(&ctl.s_full[t]);
            release_tile(2 * nxt);   // K of the next entry
          } else {
            mma_commit(&ctl.o_ready[t]);   // the stream's last P V
          }
        }
      }
      mma_commit(&ctl.o_done);
      drain_wait(&ctl.o_done, 0);   // no MMA may still run when TMEM is freed
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax streams
    const int t = (warp - 4) >> 2;           // stream of this warpgroup
    const int wq = warp & 3;                 // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;            // row inside the query tile
    const int row = q0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t sreg = tm + (t ? C::kS1 : C::kS0) + lane_off;
    const float c = kCap ? 1.f : p.c;
    const int Tt = t ? T1 : T0;
    int row_lo, row_hi;
    mod_row_keys(p.mod, row, N, row_lo, row_hi);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < Tt; ++j) {
      if (!(ok = mbar_wait_ready_first(&ctl.s_full[t], j & 1, g))) break;
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld128(sreg, sr);
      if constexpr (kCap) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          sr[i] = __float_as_uint(p.cap1 * tanh_ex2(__uint_as_float(sr[i]) * p.cap2));
      }
      const int e = ctl.tiles[2 * j + t];
      const int col0 = (e & ~kFullBit) * kBN;
      const bool need_mask = !(e & kFullBit);
      if (need_mask) {
        const int lo = row_lo - col0, hi = row_hi - col0;
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i < lo || i > hi) sr[i] = __float_as_uint(-INFINITY);
      }
      softmax_tile<D, C::kEmuPairs>(sr, need_mask, c, j, m_ref, l, sreg, sreg + C::kPOff,
                                    tm + (t ? C::kO1 : C::kO0) + lane_off, &ctl.p_half[t],
                                    &ctl.p_full[t], lane);
    }
    // ------------------------------------------------------------ merge + epilogue
    // The stream's accumulator is complete once its last P V has (all S
    // MMAs, which read the Q buffer, came before it).
    if (Tt > 0 && ok) {
      mbar_wait_ready_first(&ctl.o_ready[t], 0, g);
      tc_fence_after();
    }
    ctl.stat[t][r] = make_float2(Tt > 0 ? m_ref : -INFINITY, Tt > 0 ? l : 0.f);
    named_sync(1, 256);
    const float2 s0 = ctl.stat[0][r], s1 = ctl.stat[1][r];
    const float m = fmaxf(s0.x, s1.x);
    const float f0 = (s0.y > 0.f) ? ex2(s0.x - m) : 0.f;
    const float f1 = (s1.y > 0.f) ? ex2(s1.x - m) : 0.f;
    const float lsum = f0 * s0.y + f1 * s1.y;
    const float inv = (lsum > 0.f) ? 1.f / lsum : 0.f;
    const float w0 = f0 * inv, w1 = f1 * inv;
    // this warpgroup writes columns [t * D/2, (t + 1) * D/2) of the row,
    // from both streams' accumulators, into the Q buffer (128-byte swizzle)
    uint8_t* stage = tiles_base + C::kOffQ;
#pragma unroll
    for (int cc = 0; cc < D / 64; ++cc) {
      const int col = t * (D / 2) + cc * 32;     // first of 32 columns
      uint32_t o0[32], o1[32];
      if (T0 > 0) {
        tmem_ld32(tm + C::kO0 + lane_off + col, o0);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o0[i] = 0u;
      }
      if (T1 > 0) {
        tmem_ld32(tm + C::kO1 + lane_off + col, o1);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o1[i] = 0u;
      }
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        w[i] = pack_bf16(fmaf(__uint_as_float(o0[2 * i]), w0, __uint_as_float(o1[2 * i]) * w1),
                         fmaf(__uint_as_float(o0[2 * i + 1]), w0,
                              __uint_as_float(o1[2 * i + 1]) * w1));
      uint8_t* rowp = stage + (col >> 6) * 16384 + r * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int ch = ((col & 63) >> 3) + q;   // 16-byte chunk of the 128-byte row
        *reinterpret_cast<uint4*>(rowp + ((ch ^ (r & 7)) << 4)) =
            make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
      }
    }
    if (t == 0 && row < N)
      p.LSE[(size_t)bh * N + row] = (lsum > 0.f) ? (m + log2f(lsum)) * kLn2 : -INFINITY;
    fence_async_smem();
    named_sync(1, 256);
    if (warp == 4 && lane == 0) {
#pragma unroll
      for (int cb = 0; cb < C::kColBlocks; ++cb)
        tma_store_3d(&p.to, stage + cb * C::kBlockBytes, cb * 64, q0, bh);
      bulk_commit();
      bulk_wait_read0();   // the staging is read before the CTA exits
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

// Dynamic shared memory of one form: control block, alignment slack, tiles.
template <int D, bool kSkip>
constexpr size_t smem_bytes() {
  return sizeof(Ctl<kSkip>) + 1024 + Cfg<D, kSkip>::kOffEnd;
}
template <int D>
constexpr size_t split_smem_bytes() {
  return sizeof(CtlSplit) + 1024 + SCfg<D>::kOffEnd;
}
template <int D>
constexpr size_t persist_smem_bytes() {
  return sizeof(Ctl<false>) + 1024 + PCfg<D>::kOffEnd;
}
static_assert(smem_bytes<128, false>() <= 232448 && smem_bytes<128, true>() <= 232448 &&
                  smem_bytes<64, false>() <= 232448 && smem_bytes<64, true>() <= 232448 &&
                  persist_smem_bytes<128>() <= 232448 && persist_smem_bytes<64>() <= 232448,
              "227 KB of shared memory per CTA");

template <int D>
cudaError_t launch(const Problem& pr) {
  FwdParams kp;
  memset(&kp, 0, sizeof(kp));
  const uint64_t BHq = (uint64_t)pr.B * pr.Hq;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_seq_tmap(&kp.tq, pr, pr.Q, bf, 2, pr.Hq, 64, kBM, sw) ||
      !make_seq_tmap(&kp.tk, pr, pr.K, bf, 2, pr.Hkv, 64, kBN, sw) ||
      !make_seq_tmap(&kp.tv, pr, pr.V, bf, 2, pr.Hkv, 64, kBN, sw) ||
      !make_seq_tmap(&kp.to, pr, pr.Oout, bf, 2, pr.Hq, 64, kBM, sw))
    return cudaErrorInvalidValue;
  kp.O = static_cast<__nv_bfloat16*>(pr.Oout);
  kp.LSE = pr.LSEout;
  kp.mask = pr.mask;
  kp.err = pr.err;
  kp.N = pr.N;
  kp.Hq = pr.Hq;
  kp.Hkv = pr.Hkv;
  kp.nb = pr.nb;
  kp.nblk = (pr.N + 2 * kBM - 1) / (2 * kBM);
  kp.causal = pr.causal;
  kp.mod = mask_mod_of(pr);
  kp.c = pr.scale * kLog2e;
  const bool cap = pr.softcap > 0.f;
  kp.cap1 = cap ? pr.softcap * kLog2e : 0.f;
  kp.cap2 = cap ? pr.scale / pr.softcap : 0.f;
  kp.cu = pr.cu;
  kp.total = pr.total;
  kp.stall = debug_stall_cycles(kStallFwd);
  const size_t smem_lock = smem_bytes<D, false>(), smem_skip = smem_bytes<D, true>();
  for (const auto& fs : {std::make_pair((const void*)fwd_kernel<D, false, false, false>, smem_lock),
                         std::make_pair((const void*)fwd_kernel<D, true, false, false>, smem_lock),
                         std::make_pair((const void*)fwd_kernel<D, false, true, false>, smem_skip),
                         std::make_pair((const void*)fwd_kernel<D, false, false, true>, smem_lock),
                         std::make_pair((const void*)fwd_kernel<D, false, true, true>, smem_skip),
                         std::make_pair((const void*)fwd_persist_kernel<D, false>,
                                        persist_smem_bytes<D>()),
                         std::make_pair((const void*)fwd_split_kernel<D, false>,
                                        split_smem_bytes<D>()),
                         std::make_pair((const void*)fwd_split_kernel<D, true>,
                                        split_smem_bytes<D>()),
                         std::make_pair((const void*)fwd_persist_kernel<D, true>,
                                        persist_smem_bytes<D>())}) {
    const cudaError_t e = set_max_dynamic_smem(fs.first, (int)fs.second);
    if (e != cudaSuccess) return e;
  }
  kp.BH = (int)BHq;
  // As many heads at a time as keep their K and V within about half of the
  // 126 MB L2 (heads sharing a KV head count once): 16 for 4K-16K sequences
  // at d = 128, 4 for 64K at d = 64. Random block masks read K/V tiles out
  // of order, so a working set larger than L2 turns into DRAM re-reads.
  const uint64_t kv_bytes = 2ull * pr.N * D * 2;      // K and V of one KV head, bf16
  const uint64_t per_kv = std::max<uint64_t>(1, (64ull << 20) / kv_bytes);
  kp.chunk = (int)std::min<uint64_t>(kMaxChunk, std::max<uint64_t>(1, per_kv) * (pr.Hq / pr.Hkv));
  dim3 grid((unsigned)(BHq * kp.nblk));
  // Skip dead query-tile halves where they are common: block-sparse masks,
  // windows with a left edge and documents (variable-length batches take
  // none of them). The lockstep form walks key tiles 0 .. T-1 and relies on
  // having none.
  const bool gaps = pr.mask != nullptr || kp.mod.wl >= 0 || kp.mod.doc != nullptr;
  const bool skip = !pr.cu && gaps;
  if (!skip && gaps) return cudaErrorInvalidValue;
  if (pr.cu && cap) return cudaErrorInvalidValue;   // not offered for packed batches
  if (skip && (pr.mask != nullptr || (FA_FWD_SPLIT & 4)) && (FA_FWD_SPLIT & (D == 64 ? 1 : 2))) {
    // block-sparse: one query tile per CTA, its key tiles split between the
    // two softmax warpgroups
    const dim3 sgrid((unsigned)(BHq * (uint64_t)pr.nb));
    if (cap)
      fwd_split_kernel<D, true><<<sgrid, kThreads, split_smem_bytes<D>(), pr.stream>>>(kp);
    else
      fwd_split_kernel<D, false><<<sgrid, kThreads, split_smem_bytes<D>(), pr.stream>>>(kp);
    count_launch();
    return cudaGetLastError();
  }
  if (!pr.cu && !skip && pr.N <= FA_FWD_PERSIST_MAXN) {
    // one CTA per SM, each walking items blockIdx.x, blockIdx.x + gridDim.x, ...
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const uint64_t items = BHq * (uint64_t)kp.nblk;
    const dim3 pgrid((unsigned)std::min<uint64_t>(items, (uint64_t)std::max(sms, 1)));
    const size_t smem_p = persist_smem_bytes<D>();
    if (cap)
      fwd_persist_kernel<D, true><<<pgrid, kThreads, smem_p, pr.stream>>>(kp);
    else
      fwd_persist_kernel<D, false><<<pgrid, kThreads, smem_p, pr.stream>>>(kp);
    count_launch();
    return cudaGetLastError();
  }
  if (pr.cu)
    fwd_kernel<D, true, false, false><<<grid, kThreads, smem_lock, pr.stream>>>(kp);
  else if (skip && cap)
    fwd_kernel<D, false, true, true><<<grid, kThreads, smem_skip, pr.stream>>>(kp);
  else if (skip)
    fwd_kernel<D, false, true, false><<<grid, kThreads, smem_skip, pr.stream>>>(kp);
  else if (cap)
    fwd_kernel<D, false, false, true><<<grid, kThreads, smem_lock, pr.stream>>>(kp);
  else
    fwd_kernel<D, false, false, false><<<grid, kThreads, smem_lock, pr.stream>>>(kp);
  count_launch();
  return cudaGetLastError();
}

__global__ void exp2_fma_kernel(const float* __restrict__ x, float* __restrict__ y,
                                long long n) {
  const long long i = 2 * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float a = x[i], b = (i + 1 < n) ? x[i + 1] : 0.f;
  const float2 r = exp2_poly2(make_float2(a, b));
  y[i] = r.x;
  if (i + 1 < n) y[i + 1] = r.y;
}

}  // namespace

cudaError_t exp2_fma_eval(const float* x, float* y, long long n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const long long pairs = (n + 1) / 2;
  exp2_fma_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, stream>>>(x, y, n);
  count_launch();
  return cudaGetLastError();
}

bool sm100_fwd_supported(const Problem& p) {
  return p.dtype == 1 && (p.d == 64 || p.d == 128) && p.scale > 0.f && p.nb <= kMaxTiles &&
         (long long)p.B * p.Hq * ((p.N + 255) / 256) < (1ll << 31);
}

cudaError_t sm100_fwd(const Problem& p) {
  return p.d == 64 ? launch<64>(p) : launch<128>(p);
}

}  // namespace fa
