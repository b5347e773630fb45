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
// CTA), or skipped for it: no Q K^T, softmax or P V (kSkip: block-sparse masks
// and windows with a left edge, where a random mask makes about 40% of the
// halves dead). The skipping form counts barrier phases per query tile;
// measured on B200 it is 4-12% slower than the lockstep form where nearly
// every tile is seen by both query tiles, hence the two forms.
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 MMA issuer, warp 2
// TMEM allocator, warp 3 builds the key-tile list, warps 4-7 softmax of query
// tile 0, warps 8-11 softmax of query tile 1.
#include <math.h>

#include <algorithm>

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

template <int D>
struct Cfg {
  static constexpr int kStages = (D == 64) ? 4 : 2;
  // Share of the softmax exponentials computed on the FMA pipe, in eighths.
  // Measured on B200 (llama7b-shaped causal and 16K GQA workloads): 0 is
  // fastest here (the MUFU unit is not this kernel's bottleneck), so the
  // FMA-pipe path is compiled in but off.
  static constexpr int kEmuPairs = 0;
  static constexpr int kTileBytes = kBN * D * 2;   // one K or V tile (bf16)
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kColBlocks = D / 64;        // 128-byte column blocks per row
  static constexpr int kBlockBytes = 128 * 128;    // one column block of a 128-row tile
  static constexpr uint32_t kS0 = 0, kS1 = 128;
  static constexpr uint32_t kO0 = 256, kO1 = 256 + (D == 64 ? 64 : 128);
  static constexpr uint32_t kPOff = 64;            // P (bf16 pairs) inside S's columns
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + 2 * kQBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffEnd = kOffV + kStages * kTileBytes;
};

struct alignas(16) Ctl {
  uint64_t q_full;
  uint64_t k_full[4], v_full[4], kv_empty[4];
  uint64_t s_full[2], p_half[2], p_full[2];
  uint64_t o_ready[2];       // query tile t's last P V has completed (skipping form)
  uint64_t o_done;
  uint32_t tmem_base;
  int abort;
  int ntiles;
  int nlive[2];                  // key tiles query tile t sees (skipping form)
  uint16_t tiles[kMaxTiles];
  uint8_t dead[kMaxTiles];       // bit t: query tile t sees nothing of this key tile
  uint16_t seen[kMaxTiles][2];   // [n][t]: n-th key tile query tile t sees (skipping form)
};

struct FwdParams {
  CUtensorMap tq, tk, tv;    // [B*H][N][d] bf16, box {64, 128, 1}, 128B swizzle
  __nv_bfloat16* O;
  float* LSE;
  const uint8_t* mask;
  unsigned* err;
  int N, Hq, Hkv, nb, nblk, causal, BH;
  int wl, wr;                // visible keys: row - wl <= key <= row + wr (-1: unbounded)
  float c;                   // scale * log2(e)
  const int* cu;             // variable-length batch: sequence offsets [B+1], or null
  int total;                 // packed rows (variable-length batch)
  int chunk;                 // heads interleaved in launch order
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

// Bounded wait that ignores the abort flag (used only to drain in-flight work).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) break;
  }
}

template <int D, bool kVarlen, bool kSkip>
__global__ void __launch_bounds__(kThreads, 1) fwd_kernel(const __grid_constant__ FwdParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  Ctl& ctl = *reinterpret_cast<Ctl*>(smem_raw);
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t tile_addr = (raw_addr + sizeof(Ctl) + 1023u) & ~1023u;
  uint8_t* tiles_base = smem_raw + (tile_addr - raw_addr);

  // Heads are taken p.chunk at a time (their K/V stay in L2 during a wave);
  // inside a chunk the query blocks with the longest causal rows start first.
  int bh, rblk;
  chunked_order(blockIdx.x, p.nblk, p.BH, p.chunk, bh, rblk);
  // A launch whose error word is already set (an earlier wait ran out and
  // nobody has read the word yet) does no work: its inputs may be invalid.
  if (*reinterpret_cast<volatile unsigned*>(p.err) != 0u) return;
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

  if (threadIdx.x == 0) {
    mbar_init(&ctl.q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&ctl.k_full[s], 1);
      mbar_init(&ctl.v_full[s], 1);
      mbar_init(&ctl.kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&ctl.s_full[t], 1);
      mbar_init(&ctl.p_half[t], 4);
      mbar_init(&ctl.p_full[t], 4);
      mbar_init(&ctl.o_ready[t], 1);
    }
    mbar_init(&ctl.o_done, 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(&ctl.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 3) {
    // Key tiles either query tile can see, in increasing order.
    const int kb_end = p.wr >= 0 ? min(nb, (qb1 * kBM + kBM - 1 + p.wr) / kBN + 1) : nb;
    int count = 0, live0 = 0, live1 = 0;
    for (int kb0 = 0; kb0 < kb_end; kb0 += 32) {
      const int kb = kb0 + lane;
      bool a0 = false, a1 = false;
      if (kb < kb_end) {
        const int c0 = kb * kBN, c1 = c0 + kBN - 1;
        a0 = (!p.mask || p.mask[(size_t)qb0 * p.nb + kb]) &&
             win_any(qb0 * kBM, qb0 * kBM + kBM - 1, c0, c1, p.wl, p.wr);
        a1 = qb1 < nb && (!p.mask || p.mask[(size_t)qb1 * p.nb + kb]) &&
             win_any(qb1 * kBM, qb1 * kBM + kBM - 1, c0, c1, p.wl, p.wr);
      }
      const bool act = a0 || a1;
      const unsigned bal = __ballot_sync(0xffffffffu, act);
      if (act) {
        const int pos = count + __popc(bal & ((1u << lane) - 1u));
        ctl.tiles[pos] = static_cast<uint16_t>(kb);
        ctl.dead[pos] = static_cast<uint8_t>((a0 ? 0 : 1) | (a1 ? 0 : 2));
      }
      if constexpr (kSkip) {
        // and each query tile's own list
        const unsigned below = (1u << lane) - 1u;
        const unsigned bal0 = __ballot_sync(0xffffffffu, a0);
        const unsigned bal1 = __ballot_sync(0xffffffffu, a1);
        if (a0) ctl.seen[live0 + __popc(bal0 & below)][0] = static_cast<uint16_t>(kb);
        if (a1) ctl.seen[live1 + __popc(bal1 & below)][1] = static_cast<uint16_t>(kb);
        live0 += __popc(bal0);
        live1 += __popc(bal1);
      }
      count += __popc(bal);
    }
    if (lane == 0) {
      ctl.ntiles = count;
      ctl.nlive[0] = live0;
      ctl.nlive[1] = live1;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = ctl.tmem_base;
  const int T = ctl.ntiles;
  const Guard g{&ctl.abort, p.err};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && T > 0) {
      prefetch_tmap(&p.tq);
      prefetch_tmap(&p.tk);
      prefetch_tmap(&p.tv);
      mbar_expect_tx(&ctl.q_full, 2 * C::kQBytes);
      for (int t = 0; t < 2; ++t)
        for (int cb = 0; cb < C::kColBlocks; ++cb)
          tma_load_3d(tiles_base + C::kOffQ + t * C::kQBytes + cb * C::kBlockBytes, &p.tq,
                      &ctl.q_full, cb * 64, row0 + q0 + t * kBM, qplane);
      int issued = 0;
      for (int j = 0; j < T; ++j) {
        const int s = j % C::kStages;
        if (j >= C::kStages && !mbar_wait(&ctl.kv_empty[s], ((j / C::kStages) - 1) & 1, g))
          break;
        const int kb = ctl.tiles[j];
        mbar_expect_tx(&ctl.k_full[s], C::kTileBytes);
        for (int cb = 0; cb < C::kColBlocks; ++cb)
          tma_load_3d(tiles_base + C::kOffK + s * C::kTileBytes + cb * C::kBlockBytes, &p.tk,
                      &ctl.k_full[s], cb * 64, row0 + kb * kBN, kplane);
        mbar_expect_tx(&ctl.v_full[s], C::kTileBytes);
        for (int cb = 0; cb < C::kColBlocks; ++cb)
          tma_load_3d(tiles_base + C::kOffV + s * C::kTileBytes + cb * C::kBlockBytes, &p.tv,
                      &ctl.v_full[s], cb * 64, row0 + kb * kBN, kplane);
        issued = j + 1;
      }
      // Every issued copy has landed before the CTA may exit.
      drain_wait(&ctl.q_full, 0);
      for (int s = 0; s < C::kStages && s < issued; ++s) {
        const int n_s = (issued - 1 - s) / C::kStages + 1;  // loads into stage s
        drain_wait(&ctl.k_full[s], (n_s - 1) & 1);
        drain_wait(&ctl.v_full[s], (n_s - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && T > 0) {
      constexpr uint32_t idS = idesc_bf16(kBM, kBN, false, false);
      constexpr uint32_t idO = idesc_bf16(kBM, D, false, true);
      const uint32_t qa = smem_u32(tiles_base + C::kOffQ);
      const uint32_t ka = smem_u32(tiles_base + C::kOffK);
      const uint32_t va = smem_u32(tiles_base + C::kOffV);
      auto issue_s = [&](int t, int stage) {
        const uint32_t qt = qa + t * C::kQBytes, kt = ka + stage * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBlockBytes + (kk & 3) * 32;
          mma_ss(tm + (t ? C::kS1 : C::kS0), sdesc_sw128(qt + off, 16, 1024),
                 sdesc_sw128(kt + off, 16, 1024), idS, kk > 0);
        }
      };
      // P V over keys 64*hf .. 64*hf+63 of the tile.
      auto issue_pv = [&](int t, int stage, bool acc, int hf) {
        const uint32_t vt = va + stage * C::kTileBytes;
        const uint32_t pt = tm + (t ? C::kS1 : C::kS0) + C::kPOff;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int kk = 4 * hf + k4;
          mma_ts(tm + (t ? C::kO1 : C::kO0), pt + kk * 8,
                 sdesc_sw128(vt + kk * 16 * 128, C::kBlockBytes, 1024), idO, (acc || kk > 0));
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
        int live_next = T > 0 ? (~ctl.dead[0] & 3) : 0;
        bool ok = mbar_wait(&ctl.q_full, 0, g) && mbar_wait(&ctl.k_full[0], 0, g);
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
        }
        for (int j = 0; ok && j < T; ++j) {
          const int s = j % C::kStages;
          const uint32_t ph = (j / C::kStages) & 1;
          const bool more = j + 1 < T;
          const int s2 = (j + 1) % C::kStages;
          const int live_cur = live_next;
          live_next = more ? (~ctl.dead[j + 1] & 3) : 0;
          if (!(ok = mbar_wait(&ctl.v_full[s], ph, g))) break;
          if (live_cur & 1) {
            if (!(ok = mbar_wait(&ctl.p_half[0], n0 & 1, g))) break;
            tc_fence_after();
            issue_pv(0, s, n0 > 0, 0);
            if (!(ok = mbar_wait(&ctl.p_full[0], n0 & 1, g))) break;
            tc_fence_after();
            issue_pv(0, s, n0 > 0, 1);
            if (++n0 == nl0) mma_commit(&ctl.o_ready[0]);
          }
          if (more) {
            if (!(ok = mbar_wait(&ctl.k_full[s2], ((j + 1) / C::kStages) & 1, g))) break;
            tc_fence_after();
            if (live_next & 1) {
              issue_s(0, s2);
              mma_commit(&ctl.s_full[0]);
            }
          }
          if (live_cur & 2) {
            if (!(ok = mbar_wait(&ctl.p_half[1], n1 & 1, g))) break;
            tc_fence_after();
            issue_pv(1, s, n1 > 0, 0);
            if (!(ok = mbar_wait(&ctl.p_full[1], n1 & 1, g))) break;
            tc_fence_after();
            issue_pv(1, s, n1 > 0, 1);
            if (++n1 == nl1) mma_commit(&ctl.o_ready[1]);
          }
          mma_commit(&ctl.kv_empty[s]);
          if (more && (live_next & 2)) {
            issue_s(1, s2);
            mma_commit(&ctl.s_full[1]);
          }
        }
        // Every query tile's epilogue gets its signal, also after an abort.
        if (n0 != nl0 || nl0 == 0) mma_commit(&ctl.o_ready[0]);
        if (n1 != nl1 || nl1 == 0) mma_commit(&ctl.o_ready[1]);
      } else {
        bool ok = mbar_wait(&ctl.q_full, 0, g) && mbar_wait(&ctl.k_full[0], 0, g);
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
          mma_commit(&ctl.s_full[0]);
          issue_s(1, 0);
          mma_commit(&ctl.s_full[1]);
        }
        for (int j = 0; ok && j < T; ++j) {
          const int s = j % C::kStages;
          const uint32_t ph = (j / C::kStages) & 1;
          if (!(ok = mbar_wait(&ctl.v_full[s], ph, g) && mbar_wait(&ctl.p_half[0], j & 1, g)))
            break;
          tc_fence_after();
          issue_pv(0, s, j > 0, 0);
          if (!(ok = mbar_wait(&ctl.p_full[0], j & 1, g))) break;
          tc_fence_after();
          issue_pv(0, s, j > 0, 1);
          const bool more = j + 1 < T;
          const int s2 = (j + 1) % C::kStages;
          if (more) {
            if (!(ok = mbar_wait(&ctl.k_full[s2], ((j + 1) / C::kStages) & 1, g))) break;
            tc_fence_after();
            issue_s(0, s2);
            mma_commit(&ctl.s_full[0]);
          }
          if (!(ok = mbar_wait(&ctl.p_half[1], j & 1, g))) break;
          tc_fence_after();
          issue_pv(1, s, j > 0, 0);
          if (!(ok = mbar_wait(&ctl.p_full[1], j & 1, g))) break;
          tc_fence_after();
          issue_pv(1, s, j > 0, 1);
          mma_commit(&ctl.kv_empty[s]);
          if (more) {
            issue_s(1, s2);
            mma_commit(&ctl.s_full[1]);
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
    const float c = p.c;
    const int tile_row0 = q0 + t * kBM;
    float m_ref = -INFINITY, l = 0.f;
    // Lockstep form: every tile of the list, n = it. Skipping form: only the
    // tiles this query tile sees, it = 2n + t walking entry [n][t] of its list.
    constexpr int kStep = kSkip ? 2 : 1;
    const int it_end = kSkip ? 2 * ctl.nlive[t] + t : T;
    int it = kSkip ? t : 0;
    for (; it < it_end; it += kStep) {
      const int n = kSkip ? (it >> 1) : it;   // tiles of this query tile so far
      if (!mbar_wait(&ctl.s_full[t], n & 1, g)) break;
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld128(sreg, sr);
      const int col0 = (kSkip ? (&ctl.seen[0][0])[it] : ctl.tiles[it]) * kBN;
      const bool dead = !kSkip && ((ctl.dead[it] >> t) & 1);
      const bool need_mask = dead || col0 + kBN > N ||
                             win_cuts(tile_row0, tile_row0 + kBM - 1, col0, col0 + kBN - 1, p.wl, p.wr);
      if (need_mask) {
        // this row's visible columns of the tile: [lo, hi] relative to col0
        int lo = (p.wl >= 0) ? row - p.wl - col0 : 0;
        int hi = min(N - 1, (p.wr >= 0) ? row + p.wr : N - 1) - col0;
        if (dead) hi = lo - 1;
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i < lo || i > hi) sr[i] = __float_as_uint(-INFINITY);
      }
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
          exp_pack32<false, C::kEmuPairs>(&sr[64 * hf], c2, nmu2, acc, pk);
        else
          exp_pack32<true, C::kEmuPairs>(&sr[64 * hf], c2, nmu2, acc, pk);
        tmem_st32(sreg + C::kPOff + 32 * hf, pk);
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
          if (lane == 0) mbar_arrive(&ctl.p_half[t]);
        }
      }
      const float2 a01 = fadd2(acc[0], acc[1]), a23 = fadd2(acc[2], acc[3]);
      l += (a01.x + a01.y) + (a23.x + a23.y);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.p_full[t]);
    }
    // ------------------------------------------------------------ epilogue
    // The accumulator holds something only if some P V ran into it.
    bool have_o;
    if constexpr (kSkip)
      have_o = __any_sync(0xffffffffu, it > 1);
    else
      have_o = T > 0;
    if (have_o) {
      mbar_wait(kSkip ? &ctl.o_ready[t] : &ctl.o_done, 0, g);
      tc_fence_after();
    }
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
    const bool valid = row < N;
    // O rows: [B][H][N][d] (dense) or [total][H][d] (variable-length)
    const size_t o_base = kVarlen ? ((size_t)row0 * p.Hq + h) * D : (size_t)bh * p.N * D;
    const size_t o_rs = kVarlen ? (size_t)p.Hq * D : (size_t)D;
    const size_t lse_base = kVarlen ? (size_t)h * p.total + row0 : (size_t)bh * p.N;
    __nv_bfloat16* out = p.O + o_base + (size_t)(valid ? row : 0) * o_rs;
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
    if (valid) p.LSE[lse_base + row] = (l > 0.f) ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
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
  FwdParams kp;
  memset(&kp, 0, sizeof(kp));
  const uint64_t BHq = (uint64_t)pr.B * pr.Hq;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_seq_tmap(&kp.tq, pr, pr.Q, bf, 2, pr.Hq, 64, kBM, sw) ||
      !make_seq_tmap(&kp.tk, pr, pr.K, bf, 2, pr.Hkv, 64, kBN, sw) ||
      !make_seq_tmap(&kp.tv, pr, pr.V, bf, 2, pr.Hkv, 64, kBN, sw))
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
  // a bound of N or more cuts nothing: unbounded (keeps row +- bound in int range)
  kp.wl = (pr.wl >= pr.N) ? -1 : pr.wl;
  kp.wr = pr.causal ? 0 : ((pr.wr >= pr.N) ? -1 : pr.wr);   // causal is the window wr = 0
  kp.c = pr.scale * kLog2e;
  kp.cu = pr.cu;
  kp.total = pr.total;
  const size_t smem = sizeof(Ctl) + 1024 + C::kOffEnd;
  static bool attr_set = false;
  if (!attr_set) {
    for (const void* f : {(const void*)fwd_kernel<D, false, false>,
                          (const void*)fwd_kernel<D, false, true>,
                          (const void*)fwd_kernel<D, true, false>}) {
      const cudaError_t e =
          cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    attr_set = true;
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
  // Skip dead query-tile halves where they are common: block-sparse masks and
  // windows with a left edge (variable-length batches take neither).
  const bool skip = !pr.cu && (pr.mask != nullptr || kp.wl >= 0);
  if (pr.cu)
    fwd_kernel<D, true, false><<<grid, kThreads, smem, pr.stream>>>(kp);
  else if (skip)
    fwd_kernel<D, false, true><<<grid, kThreads, smem, pr.stream>>>(kp);
  else
    fwd_kernel<D, false, false><<<grid, kThreads, smem, pr.stream>>>(kp);
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
