// moda_fwd.cu -- fused MoDA forward for B200 (sm_100a).
//
// What it computes (hyper.ai summary of arXiv 2603.15619, sections "Mixture-of-Depths
// Attention (MoDA)" and "Hardware-efficient implementation"): for every query row, one
// online softmax state (running max m, normaliser l, fp32 accumulator O) receives the
// logits of the row's own-token depth block and of every visible causal sequence block
// before the single normalisation at the end.
//
// One CTA owns a PAIR of adjacent query tiles.  A tile is 128 rows = TQ tokens x the G
// heads of one KV group (token-major), so each K/V block and depth chunk loaded serves all
// G heads of the group ("group-aware"), and a tile reads only its own tokens' TQ x L depth
// rows ("chunk-aware"), each byte once.  Both tiles consume every K/V block the CTA loads.
//
// Two depth paths (template flag kDense), the same operator:
//   dense (default when G divides 128): a tile's depth rows go through the tensor-core
//            pipeline ahead of its sequence blocks, as extra 128-key blocks of G entries
//            of each of the tile's 128/G tokens (token-major).  Row r only sees its own
//            token's G keys, so most of each depth block's products are masked away; the
//            tensor cores have the FLOPs to spare, and the depth rows then stream through
//            the same TMA ring as K/V at the rate HBM delivers them.
//   fold:    the depth logits q.kd are computed on CUDA cores from the tile's depth
//            chunks, folded into (m, l) with the P.vd sums accumulated in registers and
//            stored into TMEM as O's starting value, before the sequence blocks.
//
// Warp roles (320 threads):
//   warps 0-3 / 4-7  tile 0 / tile 1 compute warps: thread r owns row r of its tile (TMEM
//            lane r).  Fold path: the depth fold first.  Then per block (depth blocks of
//            the dense path, then sequence blocks): S row from TMEM -> mask -> exp2 -> P
//            (bf16) back into TMEM over S; O is rescaled only when the row max grows by
//            more than 2^8.  A sequence block's P is published in two halves of 64 keys
//            (O rescaled before the first), so that the products of the first half run
//            while the warps compute the second.  Last the epilogue.
//   warp 8   TMA producer: lane 0 streams the Q tiles and the K/V blocks (dense path:
//            preceded by each depth step's kd/vd blocks of both tiles) through the K/V
//            ring; fold path: lanes 1 and 2 stream tile 0's and tile 1's depth chunks
//            through their own depth rings.  Every ring has exactly one in-order consumer.
//   warp 9   tcgen05 issuer, in the order S0(0) S1(0) { PV0(j) S0(j+1) PV1(j) S1(j+1) }
//            (each PV in two halves of 64 keys, the first after P's first half):
//            while one tile's warps turn S into P, the tensor cores work for the other
//            tile.  Because S_t(j+1) is issued after PV_t(j), a tile's warps that have
//            seen S_t(j+1) know PV_t(j) has finished, so rescaling O_t needs no extra wait.
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <type_traits>

#include "moda_internal.h"
#include "sm100.cuh"

namespace moda {

namespace {

constexpr int kBM = 128;           // rows per query tile
constexpr int kBN = 128;           // keys per sequence block
constexpr int kJCMax = 8;          // depth entries per depth chunk (max)
constexpr int kRegion = 16384;     // one 128-row x 128-byte swizzled region
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only past 256x
// In sequence blocks that need no mask, every kExpFmaPeriod-th pair of exponentials is
// computed by exp2_fma2 on the FMA pipe: at d = 128 the exponent unit is as busy as the
// tensor cores, and moving a quarter of its work off it shortens each block's softmax.
constexpr int kExpFmaPeriod = 4;

// 2^x for a pair of scores on the FMA and integer pipes, leaving the exponent unit free:
// adding 1.5 * 2^23 (whose float spacing is 1) rounds x to the nearest integer j, a cubic
// fitted for least maximum relative error gives 2^(x - j) on [-1/2, 1/2] (at most 7.5e-5
// in fp32, far inside the bf16 rounding of P), and j is added to the exponent field.  x
// is clamped below at -125, whose 2^-125 is negligible beside any row sum it joins.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  constexpr float kRound = 12582912.f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -125.f);
  x.y = fmaxf(x.y, -125.f);
  const float2 t = fadd2(x, make_float2(kRound, kRound));
  const float2 jf = fadd2(t, make_float2(-kRound, -kRound));
  const float2 f = ffma2(jf, make_float2(-1.f, -1.f), x);
  float2 p = ffma2(make_float2(0.05517132f, 0.05517132f), f,
                   make_float2(0.24261054f, 0.24261054f));
  p = ffma2(p, f, make_float2(0.69326097f, 0.69326097f));
  p = ffma2(p, f, make_float2(0.99992812f, 0.99992812f));
  // t's low mantissa bits hold j (two's complement): shifted to the exponent field they
  // add j to p's exponent, and the constant's own bits shift out
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}
constexpr int kFwdThreads = 320;

// kDense selects the depth path: false = CUDA-core fold from two depth rings, true =
// depth blocks through the K/V ring on the tensor cores (see the kernel comment).
template <int D, bool kDense>
struct FwdCfg {
  static constexpr int kRegions = D / 64;                // 64-column swizzled regions
  static constexpr int kTileBytes = kRegions * kRegion;  // one Q tile / one K or V block
  // K/V ring stages; the dense path has no depth rings and spends their room here
  static constexpr int kKV = kDense ? ((D == 128) ? 5 : 8) : ((D == 128) ? 3 : 4);
  static constexpr int kDS = kDense ? 0 : ((D == 128) ? 2 : 3);  // stages per depth ring
  static constexpr int kOffQ = 0;                        // two Q tiles
  static constexpr int kOffKV = 2 * kTileBytes;
  static constexpr int kOffD = kOffKV + kKV * kTileBytes;  // two depth rings
  static constexpr int kBarOff = kOffD + 2 * kDS * kRegion;
  static constexpr int kSmemBytes = 1024 + kBarOff + 512;
};

struct FwdArgs {
  __nv_bfloat16* out;
  float* lse;
  int B, Hq, Hkv, T, L, G, TQ, JC, nqt, npairs, causal;
  int depth_only;  // no sequence blocks: each row attends to its own token's depth only
  float scale_log2;
};

struct Bars {
  uint64_t q_full;
  uint64_t full[8];       // K/V ring: data landed
  uint64_t empty[8];      // K/V ring: stage released by the tensor cores
  uint64_t dfull[2][3];   // depth ring of tile t: data landed
  uint64_t dempty[2][3];  // depth ring of tile t: stage released by tile t's warps
  uint64_t s_full[2];     // S_t(j) in TMEM
  uint64_t p_half[2];     // keys [0, 64) of P_t(j) in TMEM, O_t rescaled (all 128 threads)
  uint64_t p_full[2];     // P_t(j) in TMEM (and O_t rescaled)
  uint64_t o_final[2];    // last PV_t done
  uint64_t drain;         // abort path: every product issued so far has finished
  uint32_t tmem_base;
  int abort;
};

// Sequence blocks between two interleaved depth steps of the dense depth path.  At 64K
// tokens (G = 4, L = 32) a depth step brings 128 KB from HBM, about twice the time of a
// sequence block's tensor work at one SM's share of the bandwidth; spacings 1 / 2 / 3 / 4
// measured 18.0 / 17.5 / 17.2 / 17.5 ms there (L = 0: 16.2 ms).
constexpr int kDepthSpacing = 3;

// Order of a tile pair's steps.  With ND depth steps, NB0 sequence blocks in tile 0 and a
// spacing R >= 1, the first K(R+1) steps (K = min(ND, NB0 / R)) repeat the pattern: one
// depth step, then R sequence blocks; then come the remaining depth steps, then the
// remaining sequence blocks.  Spreading the depth steps (HBM-bound) among the sequence
// blocks (tensor-bound) keeps both busy.  Tile 1 shares the mapping of every common step
// (its at most one extra block comes last), and every depth step comes before step
// ND + NB0.  ND = 0: step j is sequence block j.
struct StepMap {
  int ND, K, R;
  __device__ __forceinline__ bool is_depth(int j) const {
    const int P = R + 1;
    return j < K * P ? j % P == 0 : (j - K * P) < ND - K;
  }
  // depth step index or sequence block index of step j
  __device__ __forceinline__ int index(int j) const {
    const int P = R + 1;
    if (j < K * P) {
      const int q = j / P, m = j - q * P;
      return m == 0 ? q : q * R + (m - 1);
    }
    const int jj = j - K * P;
    return jj < ND - K ? K + jj : K * R + (jj - (ND - K));
  }
  // ring entries loaded before step j (4 per depth step, 2 per sequence block)
  __device__ __forceinline__ int entry(int j) const {
    const int P = R + 1;
    int nd, ns;
    if (j < K * P) {
      nd = (j + P - 1) / P;
      ns = j - nd;
    } else {
      const int jj = j - K * P;
      nd = K + min(jj, ND - K);
      ns = K * R + max(0, jj - (ND - K));
    }
    return 4 * nd + 2 * ns;
  }
};

__device__ __forceinline__ float dot8(const float (&a)[8], uint4 w) {
  float s = a[0] * bf16lo(w.x);
  s = fmaf(a[1], bf16hi(w.x), s);
  s = fmaf(a[2], bf16lo(w.y), s);
  s = fmaf(a[3], bf16hi(w.y), s);
  s = fmaf(a[4], bf16lo(w.z), s);
  s = fmaf(a[5], bf16hi(w.z), s);
  s = fmaf(a[6], bf16lo(w.w), s);
  s = fmaf(a[7], bf16hi(w.w), s);
  return s;
}

template <int D, bool kDense>
__global__ void __launch_bounds__(kFwdThreads, 1)
    moda_fwd_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmKD,
                    const __grid_constant__ CUtensorMap tmVD, const FwdArgs a) {
  using Cfg = FwdCfg<D, kDense>;
  constexpr int NKV = Cfg::kKV;
  constexpr int NDS = Cfg::kDS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s0 = smem_u32(smem);
  auto sQ = [&](int t) { return s0 + Cfg::kOffQ + uint32_t(t) * Cfg::kTileBytes; };
  auto sKV = [&](int s) { return s0 + Cfg::kOffKV + uint32_t(s) * Cfg::kTileBytes; };
  auto sDS = [&](int t, int s) { return s0 + Cfg::kOffD + uint32_t(t * NDS + s) * kRegion; };
  Bars* bars = reinterpret_cast<Bars*>(smem + Cfg::kBarOff);
  volatile int* abort_flag = &bars->abort;
  auto bar = [&](uint64_t& b) { return smem_u32(&b); };

  const int warp = threadIdx.x >> 5;
  const int nbg = a.B * a.Hkv;
  const int bg = blockIdx.x % nbg;
  const int pair = a.npairs - 1 - blockIdx.x / nbg;  // heaviest (latest) pairs first
  const int tq0 = 2 * pair * a.TQ, tq1 = tq0 + a.TQ;  // first token of tile 0 / tile 1
  const int NB0 =
      a.depth_only ? 0 : ((a.causal ? min(a.T, tq0 + a.TQ) : a.T) + kBN - 1) / kBN;
  // NB0 <= NB1; a tile 1 past the end of the sequence is computed but never stored
  const int NB1 = (tq1 >= a.T || a.depth_only)
                      ? NB0
                      : ((a.causal ? min(a.T, tq1 + a.TQ) : a.T) + kBN - 1) / kBN;
  const bool has_depth = a.L > 0;
  const int nchunk = has_depth ? (a.L + a.JC - 1) / a.JC : 0;
  const int NC = kDense ? 0 : nchunk;  // CUDA-core fold chunks
  const int ND = kDense ? nchunk : 0;  // tensor-core depth steps (ahead of the sequence)
  const int N0 = ND + NB0, N1 = ND + NB1;  // steps of tile 0 / tile 1
  constexpr int kDUses = 2 * Cfg::kRegions;   // depth stage uses per chunk: kd, vd regions
  const StepMap sm{ND, min(ND, NB0 / kDepthSpacing), kDepthSpacing};
  // Ring entries in load order.  Depth step: kd of tile 0, kd of tile 1, vd of tile 0,
  // vd of tile 1; sequence block: K then V, shared by both tiles.
  auto kidx = [&](int t, int j) { return sm.entry(j) + (sm.is_depth(j) ? t : 0); };
  auto vidx = [&](int t, int j) { return sm.entry(j) + (sm.is_depth(j) ? 2 + t : 1); };

  if (threadIdx.x == 0) {
    mbar_init(bar(bars->q_full), 1);
    for (int s = 0; s < NKV; ++s) {
      mbar_init(bar(bars->full[s]), 1);
      mbar_init(bar(bars->empty[s]), 1);
    }
    for (int t = 0; t < 2; ++t) {
      for (int s = 0; s < NDS; ++s) {
        mbar_init(bar(bars->dfull[t][s]), 1);
        mbar_init(bar(bars->dempty[t][s]), 128);
      }
      mbar_init(bar(bars->s_full[t]), 1);
      mbar_init(bar(bars->p_half[t]), 128);
      mbar_init(bar(bars->p_full[t]), 1);
      mbar_init(bar(bars->o_final[t]), 1);
    }
    mbar_init(bar(bars->drain), 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  // Rows past TQ*G (when G does not divide 128) never receive TMA data: zero them in both
  // Q tiles so the tensor cores see finite values there.
  if (threadIdx.x < kBM && threadIdx.x >= a.TQ * a.G) {
    for (int t = 0; t < 2; ++t)
      for (int rg = 0; rg < Cfg::kRegions; ++rg) {
        uint4* row = reinterpret_cast<uint4*>(smem + Cfg::kOffQ + t * Cfg::kTileBytes +
                                              rg * kRegion + threadIdx.x * 128);
        for (int c = 0; c < 8; ++c) row[c] = make_uint4(0, 0, 0, 0);
      }
    fence_proxy_async_smem();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer lanes
    const int lane = threadIdx.x & 31;
    // test-only fault: issue no loads, so that every wait for them runs out
    const bool no_loads = g_device_fault == kFaultForwardNoLoads;
    if (lane == 0 && !no_loads) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_expect_tx(bar(bars->q_full), 2 * Cfg::kRegions * 128 * a.G * a.TQ);
      for (int t = 0; t < 2; ++t)
        for (int rg = 0; rg < Cfg::kRegions; ++rg)
          tma_load_4d(sQ(t) + rg * kRegion, &tmQ, bar(bars->q_full), rg * 64, 0,
                      t ? tq1 : tq0, bg);
      int e = 0;  // ring entry
      // next ring stage, or -1 once a wait for a free stage has failed (the CTA aborts)
      auto acquire = [&](int bytes) {
        const int s = e % NKV;
        if (e >= NKV && !mbar_wait(bar(bars->empty[s]), ((e / NKV) - 1) & 1, abort_flag))
          return -1;
        mbar_expect_tx(bar(bars->full[s]), uint32_t(bytes));
        ++e;
        return s;
      };
      bool stop = false;
      for (int j = 0; j < N1 && !stop; ++j) {
        const int ix = sm.index(j);
        if (sm.is_depth(j)) {
          // depth chunk ix of each tile: entries [ix*JC, ix*JC+JC) of its TQ tokens
          for (int u = 0; u < 4 && !stop; ++u) {
            const int s = acquire(Cfg::kTileBytes);
            if (s < 0) { stop = true; break; }
            const CUtensorMap* map = (u < 2) ? &tmKD : &tmVD;
            for (int rg = 0; rg < Cfg::kRegions; ++rg)
              tma_load_4d(sKV(s) + rg * kRegion, map, bar(bars->full[s]), rg * 64,
                          ix * a.JC, (u & 1) ? tq1 : tq0, bg);
          }
        } else {
          for (int u = 0; u < 2 && !stop; ++u) {
            const int s = acquire(Cfg::kTileBytes);
            if (s < 0) { stop = true; break; }
            const CUtensorMap* map = u ? &tmV : &tmK;
            for (int rg = 0; rg < Cfg::kRegions; ++rg)
              tma_load_3d(sKV(s) + rg * kRegion, map, bar(bars->full[s]), rg * 64, ix * kBN,
                          bg);
          }
        }
      }
      if (*abort_flag) {
        // abort path: the loads issued so far still land in shared memory; wait for them
        // (Q, and the last NKV ring entries: every earlier one was consumed) before exit
        mbar_wait_drain(bar(bars->q_full), 0);
        for (int i = (e > NKV ? e - NKV : 0); i < e; ++i)
          mbar_wait_drain(bar(bars->full[i % NKV]), (i / NKV) & 1);
      }
    } else if constexpr (!kDense) if ((lane == 1 || lane == 2) && NC > 0 && !no_loads) {
      // Depth chunk ci of tile t: entries [ci*JC, ci*JC+JC) of the tile's TQ tokens as
      // rows (token, entry), one 64-column region per stage: kd regions, then vd regions.
      const int t = lane - 1;
      if (t == 0) {
        tma_prefetch_desc(&tmKD);
        tma_prefetch_desc(&tmVD);
      }
      const uint32_t dbytes = 128u * a.TQ * a.JC;
      // Each use is also pulled into L2 kDPrefetch uses ahead of its load, so the ring's
      // few shared-memory stages refill from L2 rather than from DRAM.
      constexpr int kDPrefetch = 6;
      const int nuse = NC * kDUses;
      auto box = [&](int idx, const CUtensorMap*& map, int& x, int& y) {
        const int u = idx % kDUses;
        map = (u < Cfg::kRegions) ? &tmKD : &tmVD;
        x = (u % Cfg::kRegions) * 64;
        y = (idx / kDUses) * a.JC;
      };
      for (int idx = 0; idx < kDPrefetch && idx < nuse; ++idx) {
        const CUtensorMap* map; int x, y;
        box(idx, map, x, y);
        tma_prefetch_l2_4d(map, x, y, t ? tq1 : tq0, bg);
      }
      int issued = 0;
      for (int idx = 0; idx < nuse; ++idx) {
        if (idx + kDPrefetch < nuse) {
          const CUtensorMap* pmap; int px, py;
          box(idx + kDPrefetch, pmap, px, py);
          tma_prefetch_l2_4d(pmap, px, py, t ? tq1 : tq0, bg);
        }
        const int s = idx % NDS;
        if (idx >= NDS &&
            !mbar_wait(bar(bars->dempty[t][s]), ((idx / NDS) - 1) & 1, abort_flag))
          break;
        const int u = idx % kDUses;
        const CUtensorMap* map = (u < Cfg::kRegions) ? &tmKD : &tmVD;
        const int rg = u % Cfg::kRegions;
        mbar_expect_tx(bar(bars->dfull[t][s]), dbytes);
        tma_load_4d(sDS(t, s), map, bar(bars->dfull[t][s]), rg * 64, (idx / kDUses) * a.JC,
                    t ? tq1 : tq0, bg);
        issued = idx + 1;
      }
      if (*abort_flag) {
        // abort path: wait for this ring's loads still in flight before exit
        for (int i = (issued > NDS ? issued - NDS : 0); i < issued; ++i)
          mbar_wait_drain(bar(bars->dfull[t][i % NDS]), (i / NDS) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ tcgen05 issuer
    if (elect_one()) {
      constexpr uint32_t idesc_s = make_idesc_bf16(kBM, kBN, 0, 0);
      constexpr uint32_t idesc_o = make_idesc_bf16(kBM, D, 0, 1);
      mbar_wait(bar(bars->q_full), 0, abort_flag);
      auto wait_entry = [&](int e) {
        mbar_wait(bar(bars->full[e % NKV]), (e / NKV) & 1, abort_flag);
        tc_fence_after();
      };
      auto release = [&](int e) { tc_commit(bar(bars->empty[e % NKV])); };
      // A sequence block's K and V are released after tile 1 (the last user) has read
      // them; a depth block is its tile's own.  Tile 1 does not wait again for a sequence
      // block's entries that tile 0 (same thread, earlier) already saw land: each wait is
      // a shared-memory round trip on the path from P to the next product.
      auto seen_by_tile0 = [&](int t, int j) { return t == 1 && j < N0 && !sm.is_depth(j); };
      auto issue_s = [&](int t, int j) {
        const int e = kidx(t, j);
        if (seen_by_tile0(t, j))
          tc_fence_after();
        else
          wait_entry(e);
        const uint32_t kbase = sKV(e % NKV);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks / 4) * kRegion + (ks % 4) * 32;
          mma_ss(tmem + t * 128, make_sdesc_sw128(sQ(t) + off, 16, 1024),
                 make_sdesc_sw128(kbase + off, 16, 1024), idesc_s, ks > 0 ? 1u : 0u);
        }
        tc_commit(bar(bars->s_full[t]));
        if (sm.is_depth(j) || t == 1) release(e);
      };
      auto issue_pv = [&](int t, int j) {
        const int e = vidx(t, j);
        // V's entry first: it has normally landed long before P is ready
        if (!seen_by_tile0(t, j)) wait_entry(e);
        const uint32_t vbase = sKV(e % NKV);
        const uint32_t tO = tmem + 256 + t * D;
        // keys [0, 64) as soon as their P is in (while the warps compute the rest), then
        // keys [64, 128)
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          mbar_wait(bar(part ? bars->p_full[t] : bars->p_half[t]), j & 1, abort_flag);
          tc_fence_after();
#pragma unroll
          for (int kq = 0; kq < kBN / 32; ++kq) {
            const int ks = part * (kBN / 32) + kq;
            mma_ts(tO, tmem + t * 128 + ks * 8,
                   make_sdesc_sw128(vbase + ks * 2048, kRegion, 1024), idesc_o,
                   (ks > 0 || j > 0 || NC > 0) ? 1u : 0u);
          }
        }
        if (sm.is_depth(j) || t == 1) release(e);
      };
      // (no steps at all: depth-only attention on the fold path, whose O is the fold's)
      if (N1 > 0) {
        issue_s(0, 0);
        issue_s(1, 0);
      }
      for (int j = 0; j < N1; ++j) {
        if (j < N0) {
          issue_pv(0, j);
          if (j == N0 - 1) tc_commit(bar(bars->o_final[0]));
          if (j + 1 < N0) issue_s(0, j + 1);
        }
        issue_pv(1, j);
        if (j == N1 - 1) tc_commit(bar(bars->o_final[1]));
        if (j + 1 < N1) issue_s(1, j + 1);
      }
      if (*abort_flag) {
        // abort path: let every product issued so far finish before TMEM is released
        tc_commit(bar(bars->drain));
        mbar_wait_drain(bar(bars->drain), 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ compute warps
    const int tt = warp >> 2;                     // tile of this warpgroup
    const int r = threadIdx.x & 127;              // tile row
    const int tok = r / a.G;
    const int hl = r - tok * a.G;
    const int t0 = tt ? tq1 : tq0;
    const int t = t0 + tok;
    const bool valid = (tok < a.TQ) && (t < a.T);
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + tt * 128;
    const uint32_t tO = tmem + lane_base + 256 + tt * D;
    const uint32_t q_base = sQ(tt);
    const int NS = tt ? N1 : N0;  // steps of this tile
    const uint32_t wg_bar = 1 + tt;               // named barrier of this warpgroup
    float m = -INFINITY, l = 0.f;

    mbar_wait(bar(bars->q_full), 0, abort_flag);

    if constexpr (!kDense) if (NC > 0) {
      float acc[D];
#pragma unroll
      for (int c = 0; c < D; ++c) acc[c] = 0.f;
      const int tokc = tok < a.TQ ? tok : 0;  // padding rows read a valid row
      int use = 0;
      auto take = [&]() -> uint32_t {
        const int s = use % NDS;
        mbar_wait(bar(bars->dfull[tt][s]), (use / NDS) & 1, abort_flag);
        return sDS(tt, s);
      };
      // every thread releases the stage itself (the empty barrier counts 128 arrivals),
      // so a fast thread never waits at a barrier for the slow ones of the warpgroup
      auto give = [&]() {
        mbar_arrive(bar(bars->dempty[tt][use % NDS]));
        ++use;
      };
      for (int ci = 0; ci < NC; ++ci) {
        float y[kJCMax];
#pragma unroll
        for (int jj = 0; jj < kJCMax; ++jj) y[jj] = 0.f;
#pragma unroll
        for (int rg = 0; rg < Cfg::kRegions; ++rg) {
          const uint32_t kb = take();
#pragma unroll 2
          for (int c8 = 0; c8 < 8; ++c8) {
            const uint4 qw = lds128(q_base + rg * kRegion + sw128_off(r, c8));
#pragma unroll
            for (int jj = 0; jj < kJCMax; ++jj)
              if (jj < a.JC)
                y[jj] = dot8_bf16(qw, lds128(kb + sw128_off(tokc * a.JC + jj, c8)), y[jj]);
          }
          give();
        }
        // online update over this chunk's depth logits (log2 domain)
        float mx = -INFINITY;
#pragma unroll
        for (int jj = 0; jj < kJCMax; ++jj) {
          const int j = ci * a.JC + jj;
          y[jj] = (jj < a.JC && j < a.L) ? y[jj] * a.scale_log2 : -INFINITY;
          mx = fmaxf(mx, y[jj]);
        }
        const float m_new = fmaxf(m, mx);
        const float alpha = ex2(m - m_new);
        // The weights enter the P.vd sums as bf16, the same precision the sequence part's
        // P takes into the tensor cores; l sums them unrounded, as for the sequence part.
        float ps = 0.f;
        uint16_t pb[kJCMax];
#pragma unroll
        for (int jj = 0; jj < kJCMax; ++jj) {
          const float p = ex2(y[jj] - m_new);
          pb[jj] = bf16_bits(p);
          ps += p;
        }
        l = l * alpha + ps;
        m = m_new;
#pragma unroll
        for (int rg = 0; rg < Cfg::kRegions; ++rg) {
          const uint32_t vb = take();
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8) {
            float(&ac)[8] = *reinterpret_cast<float(*)[8]>(acc + rg * 64 + c8 * 8);
#pragma unroll
            for (int e = 0; e < 8; ++e) ac[e] *= alpha;
#pragma unroll
            for (int jj = 0; jj < kJCMax; ++jj)
              if (jj < a.JC) axpy8_bf16(pb[jj], lds128(vb + sw128_off(tokc * a.JC + jj, c8)), ac);
          }
          give();
        }
      }
      // depth accumulator becomes O's starting value
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) w[e] = __float_as_uint(acc[cc * 32 + e]);
        tmem_st32(tO + cc * 32, w);
      }
      tmem_wait_st();
    }

    // ---- depth steps (dense path) and sequence blocks, in the order StepMap gives
    // A depth step's 128 keys are JC = G entries of each of the tile's TQ tokens,
    // token-major, so row r (token r / G) owns keys [r - hl, r - hl + G): all inside the
    // 32 keys of its warp's rows.  Only those 32 columns are read; P is zero elsewhere.
    const int key_lim = a.causal ? t : a.T - 1;
    // Steps before K(R+1) may be either kind; then come the remaining depth steps, then
    // sequence blocks only.  Each run has its own copy of the loop body, without the code
    // of the kind it never meets, which keeps the hot loop small.
    auto run_step = [&](const int jb, auto depth_c) {
      mbar_wait(bar(bars->s_full[tt]), jb & 1, abort_flag);
      tc_fence_after();
      // kind: 0 sequence block that needs no mask, 1 depth step, 2 either (StepMap
      // decides), 3 sequence block that may need the causal or past-the-end mask
      constexpr int kind = decltype(depth_c)::value;
      const bool dstep = kDense && (kind == 1 || (kind == 2 && sm.is_depth(jb)));
      const int ix = sm.index(jb);  // depth step or sequence block index
      uint32_t s[kBN];
      float mx = -INFINITY;  // row max on the raw scores (scale > 0); masked keys -> -inf
      if (dstep) {
        tmem_ld32(tS + 32 * (warp & 3), &s[0]);
        tmem_wait_ld();
        const int lo = (r & 31) - hl;
        const int nval = min(a.JC, a.L - ix * a.JC);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (c < lo || c >= lo + nval) s[c] = __float_as_uint(-INFINITY);
          mx = fmaxf(mx, __uint_as_float(s[c]));
        }
      } else {
        tmem_ld32(tS + 0, &s[0]);
        tmem_ld32(tS + 32, &s[32]);
        tmem_ld32(tS + 64, &s[64]);
        tmem_ld32(tS + 96, &s[96]);
        tmem_wait_ld();
        const int kbase = ix * kBN;
        const bool need_mask =
            kind != 0 && (a.causal ? (kbase + kBN - 1 > t0) : (kbase + kBN > a.T));
        if (need_mask) {
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (kbase + c > key_lim) s[c] = __float_as_uint(-INFINITY);
        }
        // two chains of three-input maxima
        float mx1 = -INFINITY;
#pragma unroll
        for (int c = 0; c < kBN; c += 4) {
          mx = fmax3(mx, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
          mx1 = fmax3(mx1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
        }
        mx = fmaxf(mx, mx1);
      }
      const float m_cand = fmaxf(m, mx * a.scale_log2);
      const bool grow = m_cand > m + kRescaleThreshold;
      const float m_new = grow ? m_cand : m;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = ex2(m - m_use);
      // O_t holds every PV_t issued so far (S_t(jb) was issued after PV_t(jb-1)).  It is
      // rescaled before the first half of P is published, since that half's PV may start
      // at once.
      const bool has_o = NC > 0 || jb > 0;
      auto rescale_o = [&]() {
        if (__any_sync(0xffffffffu, grow && has_o)) {
          const float f = grow ? alpha : 1.f;
#pragma unroll 1
          for (int cc = 0; cc < D / 16; ++cc) {
            uint32_t o[16];
            tmem_ld16(tO + cc * 16, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            tmem_st16(tO + cc * 16, o);
          }
        }
      };
      float ps0 = 0.f, ps1 = 0.f;
      if (dstep) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float p0 = ex2(fmaf(__uint_as_float(s[c]), a.scale_log2, -m_use));
          const float p1 = ex2(fmaf(__uint_as_float(s[c + 1]), a.scale_log2, -m_use));
          ps0 += p0;
          ps1 += p1;
          pk[c / 2] = pack_bf16x2(p0, p1);
        }
        uint32_t zero[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) zero[c] = 0u;
        rescale_o();
        // packed P columns [16q, 16q+16) hold keys [32q, 32q+32): this warp's are pk
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (q == (warp & 3))
            tmem_st16(tS + 16 * q, pk);
          else
            tmem_st16(tS + 16 * q, zero);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(bars->p_half[tt]));  // (the whole P: a depth step's keys interleave)
      } else {
        // p = 2^(s*scale*log2e - m): one packed FFMA feeds each pair of exp2, one packed
        // add accumulates each pair
        const float2 sl2 = make_float2(a.scale_log2, a.scale_log2);
        const float2 nm2 = make_float2(-m_use, -m_use);
        float2 ps2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const float2 x = ffma2(make_float2(__uint_as_float(s[half * 64 + c]),
                                               __uint_as_float(s[half * 64 + c + 1])),
                                   sl2, nm2);
            float2 p;
            if constexpr (kind == 0) {
              if ((c / 2) % kExpFmaPeriod == kExpFmaPeriod - 1)
                p = exp2_fma2(x);
              else
                p = make_float2(ex2(x.x), ex2(x.y));
            } else {
              p = make_float2(ex2(x.x), ex2(x.y));
            }
            ps2 = fadd2(ps2, p);
            pk[c / 2] = pack_bf16x2(p.x, p.y);
          }
          if (half == 0) {
            rescale_o();
            tmem_st32(tS, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(bars->p_half[tt]));
          } else {
            tmem_st32(tS + 32, pk);
          }
        }
        ps0 = ps2.x;
        ps1 = ps2.y;
      }
      const float ps = ps0 + ps1;
      l = l * alpha + ps;
      m = m_new;
      tmem_wait_st();
      tc_fence_before();
      named_bar_sync(wg_bar, 128);
      if (r == 0) mbar_arrive(bar(bars->p_full[tt]));
    };
    const int J0 = kDense ? min(NS, sm.K * (sm.R + 1)) : 0;
    const int J1 = kDense ? min(NS, J0 + (sm.ND - sm.K)) : 0;
    // From J1 on, step j is sequence block j - J1 + K*R.  Blocks from ix_m on may hold
    // keys past a row's token (causal) or past the end; the blocks before it need no mask.
    const int ix_m = a.causal ? (t0 + 1) / kBN : a.T / kBN;
    const int JM = min(NS, J1 + max(0, ix_m - (kDense ? sm.K * sm.R : 0)));
#pragma unroll 1
    for (int jb = 0; jb < J0; ++jb) run_step(jb, std::integral_constant<int, 2>{});
#pragma unroll 1
    for (int jb = J0; jb < J1; ++jb) run_step(jb, std::integral_constant<int, 1>{});
#pragma unroll 1
    for (int jb = J1; jb < JM; ++jb) run_step(jb, std::integral_constant<int, 0>{});
#pragma unroll 1
    for (int jb = JM; jb < NS; ++jb) run_step(jb, std::integral_constant<int, 3>{});

    // ---- epilogue
    if (NS > 0) mbar_wait(bar(bars->o_final[tt]), 0, abort_flag);
    tc_fence_after();
    const float inv_l = 1.f / l;
    const int h = (bg % a.Hkv) * a.G + hl;
    const int b = bg / a.Hkv;
    const size_t row_off = ((size_t(b) * a.Hq + h) * a.T + (valid ? t : 0)) * D;
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t o[32];
      tmem_ld32(tO + cc * 32, o);
      tmem_wait_ld();
      if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(a.out + row_off + cc * 32);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(o[v4 * 8 + 0]) * inv_l,
                            __uint_as_float(o[v4 * 8 + 1]) * inv_l);
          w.y = pack_bf16x2(__uint_as_float(o[v4 * 8 + 2]) * inv_l,
                            __uint_as_float(o[v4 * 8 + 3]) * inv_l);
          w.z = pack_bf16x2(__uint_as_float(o[v4 * 8 + 4]) * inv_l,
                            __uint_as_float(o[v4 * 8 + 5]) * inv_l);
          w.w = pack_bf16x2(__uint_as_float(o[v4 * 8 + 6]) * inv_l,
                            __uint_as_float(o[v4 * 8 + 7]) * inv_l);
          dst[v4] = w;
        }
      }
    }
    if (valid) a.lse[(size_t(b) * a.Hq + h) * a.T + t] = (m + __log2f(l)) * kLn2;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Host-side tensor map helper.
bool make_map(EncodeTiledFn encode, CUtensorMap* map, const void* base, int rank,
              const cuuint64_t* dims, const cuuint64_t* strides_bytes,
              const cuuint32_t* box) {
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base),
                      dims, strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool kDense>
cudaError_t launch_forward_d(const Problem& p, const void* q, const void* k, const void* v,
                             const void* kd, const void* vd, void* out, float* lse,
                             EncodeTiledFn encode, cudaStream_t stream, const char** why) {
  using Cfg = FwdCfg<D, kDense>;
  TileGeom tg = tile_geom(p);
  // a dense depth block is JC entries of each of the tile's TQ tokens: 128 keys
  if (kDense) tg.JC = 128 / tg.TQ;
  const cuuint64_t E = 2;  // bytes per bf16
  const cuuint64_t BG = cuuint64_t(p.B) * p.Hkv;
  CUtensorMap mQ, mK, mV, mKD, mVD;
  {
    // q viewed as [bg][t][head-in-group][c] with the head stride outer to the token
    // stride, so one box lands token-major rows (token, head) in shared memory.
    const cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(p.G), cuuint64_t(p.T), BG};
    const cuuint64_t str[3] = {cuuint64_t(p.T) * D * E, cuuint64_t(D) * E,
                               cuuint64_t(p.G) * p.T * D * E};
    const cuuint32_t box[4] = {64, cuuint32_t(p.G), cuuint32_t(tg.TQ), 1};
    if (!make_map(encode, &mQ, q, 4, dims, str, box)) {
      *why = "cuTensorMapEncodeTiled failed for q";
      return cudaErrorInvalidValue;
    }
  }
  {
    const cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(p.T), BG};
    const cuuint64_t str[2] = {cuuint64_t(D) * E, cuuint64_t(p.T) * D * E};
    const cuuint32_t box[3] = {64, 128, 1};
    if (!make_map(encode, &mK, k, 3, dims, str, box) ||
        !make_map(encode, &mV, v, 3, dims, str, box)) {
      *why = "cuTensorMapEncodeTiled failed for k/v";
      return cudaErrorInvalidValue;
    }
  }
  if (p.L > 0) {
    // kd as [bg][t][j][c]: one box lands JC entries of TQ tokens as rows (token, entry).
    const cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(p.L), cuuint64_t(p.T), BG};
    const cuuint64_t str[3] = {cuuint64_t(D) * E, cuuint64_t(p.L) * D * E,
                               cuuint64_t(p.T) * p.L * D * E};
    const cuuint32_t box[4] = {64, cuuint32_t(tg.JC), cuuint32_t(tg.TQ), 1};
    if (!make_map(encode, &mKD, kd, 4, dims, str, box) ||
        !make_map(encode, &mVD, vd, 4, dims, str, box)) {
      *why = "cuTensorMapEncodeTiled failed for kd/vd";
      return cudaErrorInvalidValue;
    }
  } else {
    mKD = mK;  // unused when L == 0
    mVD = mV;
  }
  FwdArgs args;
  args.out = static_cast<__nv_bfloat16*>(out);
  args.lse = lse;
  args.B = p.B;
  args.Hq = p.Hq;
  args.Hkv = p.Hkv;
  args.T = p.T;
  args.L = p.L;
  args.G = p.G;
  args.TQ = tg.TQ;
  args.JC = tg.JC;
  args.nqt = tg.nqt;
  args.npairs = (tg.nqt + 1) / 2;
  args.causal = p.causal;
  args.depth_only = p.depth_only;
  args.scale_log2 = p.scale * kLog2e;

  {
    cudaError_t e = cudaFuncSetAttribute(moda_fwd_kernel<D, kDense>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::kSmemBytes);
    if (e != cudaSuccess) {
      *why = "cudaFuncSetAttribute(max dynamic shared memory) failed";
      return e;
    }
  }
  const unsigned grid = unsigned(BG) * unsigned(args.npairs);
  moda_fwd_kernel<D, kDense><<<grid, kFwdThreads, Cfg::kSmemBytes, stream>>>(
      mQ, mK, mV, mKD, mVD, args);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) *why = "forward kernel launch failed";
  return e;
}

// Test only: the FMA-pipe exp2 of the forward, one pair of elements per thread.
__global__ void moda_test_exp2_fma_kernel(const float* __restrict__ x, float* __restrict__ y,
                                          int n) {
  const long long i = 2ll * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const bool two = i + 1 < n;
  const float2 r = exp2_fma2(make_float2(x[i], two ? x[i + 1] : 0.f));
  y[i] = r.x;
  if (two) y[i + 1] = r.y;
}

}  // namespace

// A dense depth block gives row r only the 32 columns of its own warp, which hold the G
// entries of the row's token only when G <= 32 (and the block is whole when G divides 128).
cudaError_t launch_test_exp2_fma(const float* x, float* y, int n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int pairs = (n + 1) / 2, threads = 256;
  moda_test_exp2_fma_kernel<<<(pairs + threads - 1) / threads, threads, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

bool dense_depth_supported(const Problem& p) { return 128 % p.G == 0 && p.G <= 32; }

bool dense_depth_default(const Problem& p) {
  return dense_depth_supported(p) && p.L >= kDenseDepthMinL;
}

cudaError_t launch_forward(const Problem& p, const void* q, const void* k, const void* v,
                           const void* kd, const void* vd, void* out, float* lse,
                           int depth_path, EncodeTiledFn encode, cudaStream_t stream,
                           const char** why) {
  const bool dense = depth_path == kDepthPathDense ||
                     (depth_path == kDepthPathAuto && dense_depth_default(p));
  if (p.d == 128)
    return dense ? launch_forward_d<128, true>(p, q, k, v, kd, vd, out, lse, encode, stream, why)
                 : launch_forward_d<128, false>(p, q, k, v, kd, vd, out, lse, encode, stream, why);
  return dense ? launch_forward_d<64, true>(p, q, k, v, kd, vd, out, lse, encode, stream, why)
               : launch_forward_d<64, false>(p, q, k, v, kd, vd, out, lse, encode, stream, why);
}

}  // namespace moda
