// Deterministic dQ for sm_100a: one CTA per 128-row query tile of one
// (batch, head) walks the key tiles the tile sees and accumulates
//
//   S   = Q K_j^T                       SS MMA -> TMEM
//   dP  = dO V_j^T                      SS MMA -> TMEM
//   P   = exp2(S * scale*log2e - LSE2)  one query row per thread (P recomputed
//   dS  = P * (dP - D)                  from the saved LSE: paper summary,
//                                       "Core Idea" item 3)
//   dQ += dS K_j                        TS MMA (dS bf16 in TMEM), fp32 in TMEM
//
// and stores scale * dQ once at the end. Every dQ element is summed by one
// CTA in key-tile order, so the result does not depend on scheduling (the
// main backward kernel, which adds dQ partials from many CTAs with fp32
// reduce-adds, is run without its dQ part when this kernel is used).
//
// TMEM: S in columns 0..127 (dS, bf16 pairs, overwrites the first 64 as the
// rows are consumed), dP in 128..255, dQ in 256..256+d. tcgen05.mma
// operations issued by one thread run in order, so S_{j+1} (issued after
// dQ_j) cannot overwrite dS_j before dQ_j has read it.
//
// Warp roles (256 threads): warp 0 TMA producer, warp 1 MMA issuer, warp 2
// TMEM allocator, warp 3 builds the key-tile list, warps 4-7 the element-wise
// step and the final store.
#include <math.h>

#include "sm100_common.cuh"

namespace fa {
namespace {
using namespace sm100;

constexpr int kBM = 128;           // query rows per CTA
constexpr int kBN = 128;           // keys per tile
constexpr int kMaxTiles = 2048;    // key tiles per sequence: N <= 262144
constexpr int kThreads = 256;
constexpr int kChunk = 16;         // heads interleaved in launch order
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
  static constexpr int kStages = (D == 64) ? 4 : 2;
  static constexpr int kTileBytes = kBN * D * 2;   // one K or V tile (bf16)
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kColBlocks = D / 64;
  static constexpr int kBlockBytes = 128 * 128;    // one 64-column block of a 128-row tile
  static constexpr uint32_t kS = 0, kDP = 128, kDQ = 256;
  static constexpr int kOffQ = 0;
  static constexpr int kOffDO = kOffQ + kQBytes;
  static constexpr int kOffK = kOffDO + kQBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffEnd = kOffV + kStages * kTileBytes;
  // the epilogue stages fp32 dQ (128 rows x D) over the Q and dO tiles
  static_assert(kOffK - kOffQ >= kBM * D * 4, "epilogue staging");
};

struct alignas(16) Ctl {
  uint64_t q_full;
  uint64_t kv_full[4], kv_empty[4];
  uint64_t sp_full, ds_ready, dq_done;
  uint64_t never;                // signalled by nothing (wait-limit test hook)
  uint32_t tmem_base;
  int abort;
  int skip;                      // the error word was set at launch: the CTA does nothing
  int ntiles;
  uint16_t tiles[kMaxTiles];     // visible key tiles, | kFullBit
};

// Flag on a key-tile entry: every (query, key) pair of the tile is visible,
// so its scores need no masking.
constexpr uint16_t kFullBit = 0x8000;

struct DqParams {
  CUtensorMap tq, tdo, tk, tv;   // [B*H][N][d] bf16, box {64, 128, 1}, 128B swizzle
  CUtensorMap tdq;               // dQ [B*Hq][N][d] grad dtype, box {128 bytes, 128}, 128B swizzle
  const float* lse2;             // [B*Hq][Npad]
  const float* dvec;             // [B*Hq][Npad]
  void* dQ;                      // [B*Hq][N][d], fp32 or bf16
  const uint8_t* mask;
  unsigned* err;
  int N, Npad, Hq, Hkv, nb, nqt, causal, BH, grad_bf16;
  MaskMod mod;                   // keys each query sees (the causal flag is its wr = 0)
  float c;                       // scale * log2(e)
  float scale;
  long long stall;               // > 0: injected wait of this many cycles (test hook)
};

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) break;
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) dq_kernel(const __grid_constant__ DqParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  Ctl& ctl = *reinterpret_cast<Ctl*>(smem_raw);
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t tile_addr = (raw_addr + sizeof(Ctl) + 1023u) & ~1023u;
  uint8_t* tiles_base = smem_raw + (tile_addr - raw_addr);

  // Heads kChunk at a time; inside a chunk the query tiles with the most key
  // tiles (the last ones under the causal flag) start first.
  int bh, rqt;
  chunked_order(blockIdx.x, p.nqt, p.BH, kChunk, bh, rqt);
  // A launch whose error word is already set does no work; one thread reads
  // the word and the whole CTA leaves together, before any barrier is
  // initialised or TMEM allocated.
  if (threadIdx.x == 0) ctl.skip = (*reinterpret_cast<volatile unsigned*>(p.err) != 0u) ? 1 : 0;
  __syncthreads();
  if (ctl.skip) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = p.nqt - 1 - rqt;
  const int q0 = qt * kBM;
  const int h = bh % p.Hq, b = bh / p.Hq;
  const int bhk = b * p.Hkv + h / (p.Hq / p.Hkv);
  const int N = p.N;

  if (threadIdx.x == 0) {
    mbar_init(&ctl.q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&ctl.kv_full[s], 1);
      mbar_init(&ctl.kv_empty[s], 1);
    }
    mbar_init(&ctl.sp_full, 1);
    mbar_init(&ctl.ds_ready, 4);
    mbar_init(&ctl.dq_done, 1);
    mbar_init(&ctl.never, 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(&ctl.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 3) {
    // Key tiles this query tile sees, in increasing order (entries flagged
    // kFullBit are seen whole).
    const int kb_end = min(p.nb, mod_last_key(p.mod, q0 + kBM - 1, N) / kBN + 1);
    int count = 0;
    for (int kb0 = 0; kb0 < kb_end; kb0 += 32) {
      const int kb = kb0 + lane;
      int cls = kTileEmpty;
      if (kb < kb_end && (!p.mask || p.mask[(size_t)qt * p.nb + kb]))
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
  const int T = ctl.ntiles;
  const Guard g{&ctl.abort, p.err};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && T > 0) {
      prefetch_tmap(&p.tq);
      prefetch_tmap(&p.tdo);
      prefetch_tmap(&p.tk);
      prefetch_tmap(&p.tv);
      mbar_expect_tx(&ctl.q_full, 2 * C::kQBytes);
      for (int cb = 0; cb < C::kColBlocks; ++cb) {
        tma_load_3d(tiles_base + C::kOffQ + cb * C::kBlockBytes, &p.tq, &ctl.q_full, cb * 64, q0,
                    bh);
        tma_load_3d(tiles_base + C::kOffDO + cb * C::kBlockBytes, &p.tdo, &ctl.q_full, cb * 64,
                    q0, bh);
      }
      int issued = 0;
      for (int j = 0; j < T; ++j) {
        const int s = j % C::kStages;
        if (j >= C::kStages && !mbar_wait(&ctl.kv_empty[s], ((j / C::kStages) - 1) & 1, g))
          break;
        const int kb = ctl.tiles[j] & ~kFullBit;
        mbar_expect_tx(&ctl.kv_full[s], 2 * C::kTileBytes);
        for (int cb = 0; cb < C::kColBlocks; ++cb) {
          tma_load_3d(tiles_base + C::kOffK + s * C::kTileBytes + cb * C::kBlockBytes, &p.tk,
                      &ctl.kv_full[s], cb * 64, kb * kBN, bhk);
          tma_load_3d(tiles_base + C::kOffV + s * C::kTileBytes + cb * C::kBlockBytes, &p.tv,
                      &ctl.kv_full[s], cb * 64, kb * kBN, bhk);
        }
        issued = j + 1;
      }
      drain_wait(&ctl.q_full, 0);
      for (int s = 0; s < C::kStages && s < issued; ++s)
        drain_wait(&ctl.kv_full[s], ((issued - 1 - s) / C::kStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && T > 0) {
      constexpr uint32_t idS = idesc_bf16(kBM, kBN, false, false);
      constexpr uint32_t idQ = idesc_bf16(kBM, D, false, true);
      // base descriptors, built once; each operand is one plus a byte offset
      const uint64_t dQd = sdesc_sw128(smem_u32(tiles_base + C::kOffQ), 16, 1024);
      const uint64_t dOd = sdesc_sw128(smem_u32(tiles_base + C::kOffDO), 16, 1024);
      const uint64_t dKd = sdesc_sw128(smem_u32(tiles_base + C::kOffK), 16, 1024);
      const uint64_t dVd = sdesc_sw128(smem_u32(tiles_base + C::kOffV), 16, 1024);
      const uint64_t dKn = sdesc_sw128(smem_u32(tiles_base + C::kOffK), C::kBlockBytes, 1024);
      // X Y^T over d for X in {Q, dO} (128 x d) and Y in {K_j, V_j} (128 x d)
      auto issue_xy = [&](uint32_t dst, uint64_t xd, uint64_t yd) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBlockBytes + (kk & 3) * 32;
          mma_ss(tm + dst, sdesc_at(xd, off), sdesc_at(yd, off), idS, kk > 0);
        }
      };
      bool ok = injected_stall(&ctl.never, p.stall, g) && mbar_wait(&ctl.q_full, 0, g);
      for (int j = 0; ok && j < T; ++j) {
        const int s = j % C::kStages;
        if (!(ok = mbar_wait(&ctl.kv_full[s], (j / C::kStages) & 1, g))) break;
        tc_fence_after();
        const uint32_t so = s * C::kTileBytes;
        issue_xy(C::kS, dQd, sdesc_at(dKd, so));    // S = Q K_j^T
        issue_xy(C::kDP, dOd, sdesc_at(dVd, so));   // dP = dO V_j^T
        mma_commit(&ctl.sp_full);
        if (!(ok = mbar_wait(&ctl.ds_ready, j & 1, g))) break;
        tc_fence_after();
        // dQ += dS K_j (dS bf16 pairs in S's first 64 columns; K_j N-major)
        const uint64_t kn = sdesc_at(dKn, so);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_ts(tm + C::kDQ, tm + C::kS + kk * 8, sdesc_at(kn, kk * 16 * 128), idQ,
                 (j > 0 || kk > 0));
        mma_commit(&ctl.kv_empty[s]);
      }
      mma_commit(&ctl.dq_done);
      drain_wait(&ctl.dq_done, 0);   // no MMA may still run when TMEM is freed
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ dS, then the dQ store
    const int wq = warp & 3;
    const int r = wq * 32 + lane;            // query row inside the tile
    const int row = q0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float c = p.c;
    const size_t vrow = (size_t)bh * p.Npad + row;   // padded: row < Npad always
    const float lse2 = p.lse2[vrow], dd = p.dvec[vrow];
    // this row's visible keys: [klo, khi] (empty past N)
    int klo, khi;
    mod_row_keys(p.mod, row, N, klo, khi);
    if (row >= N) khi = -1;
    for (int j = 0; j < T; ++j) {
      if (!mbar_wait(&ctl.sp_full, j & 1, g)) break;
      tc_fence_after();
      const int ent = ctl.tiles[j];
      const int col0 = (ent & ~kFullBit) * kBN;
      const bool need_mask = !(ent & kFullBit);
#pragma unroll 1
      for (int ck = 0; ck < kBN / 32; ++ck) {
        uint32_t sv[32], dp[32];
        tmem_ld32x2(tm + C::kS + lane_off + ck * 32, tm + C::kDP + lane_off + ck * 32, sv, dp);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float p0 = ex2(fmaf(__uint_as_float(sv[e]), c, -lse2));
          float p1 = ex2(fmaf(__uint_as_float(sv[e + 1]), c, -lse2));
          if (need_mask) {
            const int k0 = col0 + ck * 32 + e;
            if (k0 < klo || k0 > khi) p0 = 0.f;
            if (k0 + 1 < klo || k0 + 1 > khi) p1 = 0.f;
          }
          pk[e >> 1] = pack_bf16(p0 * (__uint_as_float(dp[e]) - dd),
                                 p1 * (__uint_as_float(dp[e + 1]) - dd));
        }
        // dS of chunk ck into S columns 16ck..16ck+15 (already read: 16ck < 32ck + 32)
        tmem_st16(tm + C::kS + lane_off + ck * 16, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.ds_ready);
    }
    if (T > 0) {
      mbar_wait(&ctl.dq_done, 0, g);
      tc_fence_after();
    }
    // scale * dQ through the shared memory of the Q and dO tiles (every MMA
    // has completed), in the TMA's 128-byte-swizzled layout (box b of 128
    // bytes per row at b * 16 KB, row r at r * 128, 16-byte chunk c at
    // ((c ^ (r & 7)) << 4)), then TMA stores of whole lines; rows at or past
    // N are clipped by the tensor map. tcgen05.ld is warp-collective: every
    // lane loads.
    uint8_t* st = tiles_base + C::kOffQ;
#pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t v[32];
      if (T > 0) {
        tmem_ld32(tm + C::kDQ + lane_off + cc * 32, v);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      if (p.grad_bf16) {
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16(__uint_as_float(v[2 * e]) * p.scale,
                           __uint_as_float(v[2 * e + 1]) * p.scale);
        uint8_t* rowp = st + (cc >> 1) * 16384 + r * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c = 4 * (cc & 1) + q;
          *reinterpret_cast<uint4*>(rowp + ((c ^ (r & 7)) << 4)) =
              make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
      } else {
        uint8_t* rowp = st + cc * 16384 + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<float4*>(rowp + ((c ^ (r & 7)) << 4)) =
              make_float4(__uint_as_float(v[4 * c]) * p.scale, __uint_as_float(v[4 * c + 1]) * p.scale,
                          __uint_as_float(v[4 * c + 2]) * p.scale,
                          __uint_as_float(v[4 * c + 3]) * p.scale);
      }
    }
    fence_async_smem();
    named_sync(1, 128);
    if (warp == 4 && lane == 0) {
      const int esz = p.grad_bf16 ? 2 : 4;
      const int boxes = D * esz / 128, box_cols = 128 / esz;
      for (int bx = 0; bx < boxes; ++bx)
        tma_store_3d(&p.tdq, st + bx * 16384, bx * box_cols, q0, bh);
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

template <int D>
cudaError_t launch(const Problem& pr) {
  using C = Cfg<D>;
  DqParams kp;
  memset(&kp, 0, sizeof(kp));
  const uint64_t BHq = (uint64_t)pr.B * pr.Hq, BHk = (uint64_t)pr.B * pr.Hkv;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_tmap_3d(&kp.tq, pr.Q, bf, 2, D, pr.N, BHq, 64, kBM, sw) ||
      !make_tmap_3d(&kp.tdo, pr.dO, bf, 2, D, pr.N, BHq, 64, kBM, sw) ||
      !make_tmap_3d(&kp.tk, pr.K, bf, 2, D, pr.N, BHk, 64, kBN, sw) ||
      !make_tmap_3d(&kp.tv, pr.V, bf, 2, D, pr.N, BHk, 64, kBN, sw))
    return cudaErrorInvalidValue;
  {
    const bool gb = pr.grad_dtype == 1;
    const int es = gb ? 2 : 4;
    if (!make_tmap_3d(&kp.tdq, pr.dQ, gb ? bf : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, es, D, pr.N, BHq,
                      128 / es, kBM, sw))
      return cudaErrorInvalidValue;
  }
  kp.lse2 = pr.LSE2ws;
  kp.dvec = pr.Dws;
  kp.dQ = pr.dQ;
  kp.mask = pr.mask;
  kp.err = pr.err;
  kp.N = pr.N;
  kp.Npad = pr.Npad;
  kp.Hq = pr.Hq;
  kp.Hkv = pr.Hkv;
  kp.nb = pr.nb;
  kp.nqt = pr.nb;   // 128-row query tiles
  kp.causal = pr.causal;
  kp.mod = mask_mod_of(pr);
  kp.BH = (int)BHq;
  kp.grad_bf16 = pr.grad_dtype == 1;
  kp.c = pr.scale * kLog2e;
  kp.scale = pr.scale;
  kp.stall = debug_stall_cycles(kStallDq);
  const size_t smem = sizeof(Ctl) + 1024 + C::kOffEnd;
  {
    const cudaError_t e = set_max_dynamic_smem((const void*)dq_kernel<D>, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((unsigned)(BHq * kp.nqt));
  dq_kernel<D><<<grid, kThreads, smem, pr.stream>>>(kp);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

bool sm100_dq_supported(const Problem& p) {
  return p.dtype == 1 && (p.d == 64 || p.d == 128) && p.scale > 0.f && p.nb <= kMaxTiles &&
         (long long)p.B * p.Hq * p.nb < (1ll << 31) && p.cu == nullptr;
}

cudaError_t sm100_dq(const Problem& p) { return p.d == 64 ? launch<64>(p) : launch<128>(p); }

}  // namespace fa
