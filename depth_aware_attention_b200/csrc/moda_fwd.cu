// moda_fwd.cu -- fused MoDA forward for B200 (sm_100a).
//
// What it computes (hyper.ai summary of arXiv 2603.15619, sections "Mixture-of-Depths
// Attention (MoDA)" and "Hardware-efficient implementation"): for every query row, one
// online softmax state (running max m, normaliser l, fp32 accumulator O) receives the
// logits of the row's own-token depth block and of every visible causal sequence block
// before the single normalisation at the end.
//
// One CTA owns one query tile of 128 rows = TQ tokens x G heads of one KV group
// (token-major), so each K/V block and each depth chunk it loads serves all G heads of
// the group ("group-aware") and the tile touches only its own tokens' depth rows
// (TQ x L of them -- "chunk-aware"), read once from HBM.
//
// Warp roles (224 threads):
//   warps 0-3  softmax/depth/epilogue: thread r owns tile row r (TMEM lane r).
//              1. depth fold: logits q.kd and the running sums over the tile's depth
//                 chunks on CUDA cores, accumulator written into TMEM as O's start;
//              2. per sequence block: S row from TMEM -> mask -> exp2 -> P (bf16) back
//                 into TMEM over S; rescales O only when the row max grows by > 2^8;
//              3. epilogue: O / l -> bf16 out, lse = ln(sum exp).
//   warp 4     TMA producer: Q tile, then the K/V blocks through the K/V ring.
//   warp 6     TMA producer: the tile's depth chunks (kd, vd) through the depth ring.
//              Each ring has exactly one consumer (tensor cores / softmax warps), which
//              waits on every stage use in order, so the parity waits are unambiguous.
//   warp 5     tcgen05 issuer: S = Q K^T (both operands in shared memory) and
//              O += P V (P from tensor memory, V in shared memory), fp32 in TMEM.
// TMEM columns: S/P double buffer at [0,128) and [128,256), O at [256, 256+D).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

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
constexpr int kFwdThreads = 224;           // 7 warps, roles below

template <int D>
struct FwdCfg {
  static constexpr int kRegions = D / 64;                 // 64-column swizzled regions
  static constexpr int kTileBytes = kRegions * kRegion;   // Q tile or one ring stage
  static constexpr int kKV = (D == 128) ? 4 : 6;          // K/V ring stages
  static constexpr int kDS = (D == 128) ? 2 : 4;          // depth ring stages
  static constexpr int kBarOff = kTileBytes * (1 + kKV + kDS);
  static constexpr int kSmemBytes = 1024 + kBarOff + 256;
};

struct FwdArgs {
  __nv_bfloat16* out;
  float* lse;
  int B, Hq, Hkv, T, L, G, TQ, JC, nqt, causal;
  float scale_log2;
};

// Shared-memory barrier block (after the tiles).
struct Bars {
  uint64_t q_full;
  uint64_t full[6];    // K/V ring: data landed
  uint64_t empty[6];   // K/V ring: stage released by the tensor cores
  uint64_t dfull[4];   // depth ring: data landed
  uint64_t dempty[4];  // depth ring: stage released by the softmax warps
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done;
  uint64_t o_final;
  uint32_t tmem_base;
  int abort;
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

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    moda_fwd_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmKD,
                    const __grid_constant__ CUtensorMap tmVD, const FwdArgs a) {
  using Cfg = FwdCfg<D>;
  constexpr int NKV = Cfg::kKV;
  constexpr int NDS = Cfg::kDS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sRing = sQ + Cfg::kTileBytes;               // K/V ring
  const uint32_t sDRing = sRing + NKV * Cfg::kTileBytes;      // depth ring
  Bars* bars = reinterpret_cast<Bars*>(smem + Cfg::kBarOff);
  volatile int* abort_flag = &bars->abort;

  const int warp = threadIdx.x >> 5;
  const int nbg = a.B * a.Hkv;
  const int bg = blockIdx.x % nbg;
  const int qt = a.nqt - 1 - blockIdx.x / nbg;  // heaviest (latest) tiles first
  const int t0 = qt * a.TQ;
  const int kv_end = a.causal ? min(a.T, t0 + a.TQ) : a.T;
  const int NB = (kv_end + kBN - 1) / kBN;
  const int NC = a.L > 0 ? (a.L + a.JC - 1) / a.JC : 0;
  const bool has_depth = NC > 0;

  auto bar = [&](uint64_t& b) { return smem_u32(&b); };
  auto stage_addr = [&](int s) { return sRing + uint32_t(s) * Cfg::kTileBytes; };
  auto dstage_addr = [&](int s) { return sDRing + uint32_t(s) * Cfg::kTileBytes; };

  if (threadIdx.x == 0) {
    mbar_init(bar(bars->q_full), 1);
    for (int s = 0; s < NKV; ++s) {
      mbar_init(bar(bars->full[s]), 1);
      mbar_init(bar(bars->empty[s]), 1);
    }
    for (int s = 0; s < NDS; ++s) {
      mbar_init(bar(bars->dfull[s]), 1);
      mbar_init(bar(bars->dempty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(bars->s_full[i]), 1);
      mbar_init(bar(bars->p_full[i]), 1);
    }
    mbar_init(bar(bars->o_done), 1);
    mbar_init(bar(bars->o_final), 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  // Rows past TQ*G (when G does not divide 128) never receive TMA data: zero them so the
  // tensor cores see finite values there.
  if (threadIdx.x < kBM && threadIdx.x >= a.TQ * a.G) {
    for (int rg = 0; rg < Cfg::kRegions; ++rg) {
      uint4* row = reinterpret_cast<uint4*>(smem + rg * kRegion + threadIdx.x * 128);
      for (int c = 0; c < 8; ++c) row[c] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 4) {
    // ------------------------------------------------ TMA producer: Q tile, K/V blocks
    if (elect_one()) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_expect_tx(bar(bars->q_full), Cfg::kRegions * 128 * a.G * a.TQ);
      for (int rg = 0; rg < Cfg::kRegions; ++rg)
        tma_load_4d(sQ + rg * kRegion, &tmQ, bar(bars->q_full), rg * 64, 0, t0, bg);
      for (int idx = 0; idx < 2 * NB; ++idx) {
        const int s = idx % NKV;
        if (idx >= NKV) mbar_wait(bar(bars->empty[s]), ((idx / NKV) - 1) & 1, abort_flag);
        const CUtensorMap* map = (idx & 1) ? &tmV : &tmK;
        mbar_expect_tx(bar(bars->full[s]), Cfg::kTileBytes);
        for (int rg = 0; rg < Cfg::kRegions; ++rg)
          tma_load_3d(stage_addr(s) + rg * kRegion, map, bar(bars->full[s]), rg * 64,
                      (idx >> 1) * kBN, bg);
      }
    }
    __syncwarp();
  } else if (warp == 6) {
    // ------------------------------------------------ TMA producer: depth chunks
    // Chunk ci holds entries [ci*JC, ci*JC+JC) of the tile's TQ tokens, rows
    // (token, entry) with the entry fastest: each token's entries are one contiguous
    // run of the [B,Hkv,T,L,d] cache.
    if (has_depth && elect_one()) {
      tma_prefetch_desc(&tmKD);
      tma_prefetch_desc(&tmVD);
      const uint32_t dbytes = Cfg::kRegions * 128 * a.TQ * a.JC;
      for (int idx = 0; idx < 2 * NC; ++idx) {
        const int s = idx % NDS;
        if (idx >= NDS) mbar_wait(bar(bars->dempty[s]), ((idx / NDS) - 1) & 1, abort_flag);
        const CUtensorMap* map = (idx & 1) ? &tmVD : &tmKD;
        mbar_expect_tx(bar(bars->dfull[s]), dbytes);
        for (int rg = 0; rg < Cfg::kRegions; ++rg)
          tma_load_4d(dstage_addr(s) + rg * kRegion, map, bar(bars->dfull[s]), rg * 64,
                      (idx >> 1) * a.JC, t0, bg);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ tcgen05 issuer
    if (elect_one()) {
      constexpr uint32_t idesc_s = make_idesc_bf16(kBM, kBN, 0, 0);
      constexpr uint32_t idesc_o = make_idesc_bf16(kBM, D, 0, 1);
      const uint32_t tO = tmem + 256;
      mbar_wait(bar(bars->q_full), 0, abort_flag);
      auto issue_pv = [&](int j) {
        mbar_wait(bar(bars->p_full[j & 1]), (j >> 1) & 1, abort_flag);
        const int vidx = 2 * j + 1;
        const int vs = vidx % NKV;
        mbar_wait(bar(bars->full[vs]), (vidx / NKV) & 1, abort_flag);
        tc_fence_after();
        const uint32_t vbase = stage_addr(vs);
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks) {
          const uint64_t bdesc = make_sdesc_sw128(vbase + ks * 2048, kRegion, 1024);
          mma_ts(tO, tmem + (j & 1) * 128 + ks * 8, bdesc, idesc_o,
                 (ks > 0 || j > 0 || has_depth) ? 1u : 0u);
        }
        tc_commit(bar(bars->empty[vs]));
        tc_commit(bar(bars->o_done));
        if (j == NB - 1) tc_commit(bar(bars->o_final));
      };
      for (int jb = 0; jb < NB; ++jb) {
        const int kidx = 2 * jb;
        const int ks_ = kidx % NKV;
        mbar_wait(bar(bars->full[ks_]), (kidx / NKV) & 1, abort_flag);
        tc_fence_after();
        const uint32_t kbase = stage_addr(ks_);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks / 4) * kRegion + (ks % 4) * 32;
          const uint64_t adesc = make_sdesc_sw128(sQ + off, 16, 1024);
          const uint64_t bdesc = make_sdesc_sw128(kbase + off, 16, 1024);
          mma_ss(tmem + (jb & 1) * 128, adesc, bdesc, idesc_s, ks > 0 ? 1u : 0u);
        }
        tc_commit(bar(bars->s_full[jb & 1]));
        tc_commit(bar(bars->empty[ks_]));
        if (jb >= 1) issue_pv(jb - 1);
      }
      issue_pv(NB - 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps 0-3
    const int r = threadIdx.x;
    const int tok = r / a.G;
    const int hl = r - tok * a.G;
    const int t = t0 + tok;
    const bool valid = (tok < a.TQ) && (t < a.T);
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const uint32_t tO = tmem + lane_base + 256;
    float m = -INFINITY, l = 0.f;

    mbar_wait(bar(bars->q_full), 0, abort_flag);

    if (has_depth) {
      float acc[D];
#pragma unroll
      for (int c = 0; c < D; ++c) acc[c] = 0.f;
      const int tokc = tok < a.TQ ? tok : 0;  // padding rows read a valid row
      for (int ci = 0; ci < NC; ++ci) {
        const int kidx = 2 * ci, vidx = 2 * ci + 1;
        const int kst = kidx % NDS, vst = vidx % NDS;
        float y[kJCMax];
#pragma unroll
        for (int jj = 0; jj < kJCMax; ++jj) y[jj] = 0.f;
        mbar_wait(bar(bars->dfull[kst]), (kidx / NDS) & 1, abort_flag);
        const uint32_t kb = dstage_addr(kst);
#pragma unroll 2
        for (int c8 = 0; c8 < D / 8; ++c8) {
          const uint32_t reg = (c8 >> 3) * kRegion;
          const uint4 qw = lds128(sQ + reg + sw128_off(r, c8 & 7));
          float qf[8] = {bf16lo(qw.x), bf16hi(qw.x), bf16lo(qw.y), bf16hi(qw.y),
                         bf16lo(qw.z), bf16hi(qw.z), bf16lo(qw.w), bf16hi(qw.w)};
#pragma unroll
          for (int jj = 0; jj < kJCMax; ++jj) {
            if (jj < a.JC) {
              const uint32_t row = tokc * a.JC + jj;
              y[jj] += dot8(qf, lds128(kb + reg + sw128_off(row, c8 & 7)));
            }
          }
        }
        named_bar_sync(1, 128);
        if (r == 0) mbar_arrive(bar(bars->dempty[kst]));
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
        float ps = 0.f;
#pragma unroll
        for (int jj = 0; jj < kJCMax; ++jj) {
          y[jj] = ex2(y[jj] - m_new);
          ps += y[jj];
        }
        l = l * alpha + ps;
        m = m_new;
        mbar_wait(bar(bars->dfull[vst]), (vidx / NDS) & 1, abort_flag);
        const uint32_t vb = dstage_addr(vst);
#pragma unroll
        for (int c8 = 0; c8 < D / 8; ++c8) {
          const uint32_t reg = (c8 >> 3) * kRegion;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[c8 * 8 + e] *= alpha;
#pragma unroll
          for (int jj = 0; jj < kJCMax; ++jj) {
            if (jj < a.JC) {
              const uint32_t row = tokc * a.JC + jj;
              const uint4 w = lds128(vb + reg + sw128_off(row, c8 & 7));
              const float p = y[jj];
              acc[c8 * 8 + 0] = fmaf(p, bf16lo(w.x), acc[c8 * 8 + 0]);
              acc[c8 * 8 + 1] = fmaf(p, bf16hi(w.x), acc[c8 * 8 + 1]);
              acc[c8 * 8 + 2] = fmaf(p, bf16lo(w.y), acc[c8 * 8 + 2]);
              acc[c8 * 8 + 3] = fmaf(p, bf16hi(w.y), acc[c8 * 8 + 3]);
              acc[c8 * 8 + 4] = fmaf(p, bf16lo(w.z), acc[c8 * 8 + 4]);
              acc[c8 * 8 + 5] = fmaf(p, bf16hi(w.z), acc[c8 * 8 + 5]);
              acc[c8 * 8 + 6] = fmaf(p, bf16lo(w.w), acc[c8 * 8 + 6]);
              acc[c8 * 8 + 7] = fmaf(p, bf16hi(w.w), acc[c8 * 8 + 7]);
            }
          }
        }
        named_bar_sync(1, 128);
        if (r == 0) mbar_arrive(bar(bars->dempty[vst]));
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

    // ---- sequence blocks
    const int key_lim = a.causal ? t : a.T - 1;
    for (int jb = 0; jb < NB; ++jb) {
      mbar_wait(bar(bars->s_full[jb & 1]), (jb >> 1) & 1, abort_flag);
      tc_fence_after();
      const uint32_t tS = tmem + lane_base + (jb & 1) * 128;
      uint32_t s[kBN];
      tmem_ld32(tS + 0, &s[0]);
      tmem_ld32(tS + 32, &s[32]);
      tmem_ld32(tS + 64, &s[64]);
      tmem_ld32(tS + 96, &s[96]);
      tmem_wait_ld();
      const int kbase = jb * kBN;
      const bool need_mask = a.causal ? (kbase + kBN - 1 > t0) : (kbase + kBN > a.T);
      float x[kBN];
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kBN; ++c) {
        float v = __uint_as_float(s[c]) * a.scale_log2;
        if (need_mask && kbase + c > key_lim) v = -INFINITY;
        x[c] = v;
        mx = fmaxf(mx, v);
      }
      const float m_cand = fmaxf(m, mx);
      const bool grow = m_cand > m + kRescaleThreshold;
      const float m_new = grow ? m_cand : m;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = ex2(m - m_use);
      float ps = 0.f;
      uint32_t pk[kBN / 2];
#pragma unroll
      for (int c = 0; c < kBN; c += 2) {
        const float p0 = ex2(x[c] - m_use);
        const float p1 = ex2(x[c + 1] - m_use);
        ps += p0 + p1;
        pk[c / 2] = pack_bf16x2(p0, p1);
      }
      tmem_st32(tS + 0, &pk[0]);
      tmem_st32(tS + 32, &pk[32]);
      l = l * alpha + ps;
      m = m_new;
      const bool has_o = has_depth || jb > 0;
      if (__any_sync(0xffffffffu, grow && has_o)) {
        if (jb > 0) mbar_wait(bar(bars->o_done), (jb - 1) & 1, abort_flag);
        tc_fence_after();
        const float f = grow ? alpha : 1.f;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + cc * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
          tmem_st32(tO + cc * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      named_bar_sync(1, 128);
      if (r == 0) mbar_arrive(bar(bars->p_full[jb & 1]));
    }

    // ---- epilogue
    mbar_wait(bar(bars->o_final), 0, abort_flag);
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
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Host-side tensor map helpers.
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

template <int D>
cudaError_t launch_forward_d(const Problem& p, const void* q, const void* k, const void* v,
                             const void* kd, const void* vd, void* out, float* lse,
                             EncodeTiledFn encode, cudaStream_t stream, const char** why) {
  using Cfg = FwdCfg<D>;
  const TileGeom tg = tile_geom(p);
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
  args.causal = p.causal;
  args.scale_log2 = p.scale * kLog2e;

  {
    cudaError_t e = cudaFuncSetAttribute(moda_fwd_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::kSmemBytes);
    if (e != cudaSuccess) {
      *why = "cudaFuncSetAttribute(max dynamic shared memory) failed";
      return e;
    }
  }
  const unsigned grid = unsigned(BG) * unsigned(tg.nqt);
  moda_fwd_kernel<D><<<grid, kFwdThreads, Cfg::kSmemBytes, stream>>>(mQ, mK, mV, mKD, mVD, args);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) *why = "forward kernel launch failed";
  return e;
}

}  // namespace

cudaError_t launch_forward(const Problem& p, const void* q, const void* k, const void* v,
                           const void* kd, const void* vd, void* out, float* lse,
                           EncodeTiledFn encode, cudaStream_t stream, const char** why) {
  if (p.d == 128)
    return launch_forward_d<128>(p, q, k, v, kd, vd, out, lse, encode, stream, why);
  return launch_forward_d<64>(p, q, k, v, kd, vd, out, lse, encode, stream, why);
}

}  // namespace moda
